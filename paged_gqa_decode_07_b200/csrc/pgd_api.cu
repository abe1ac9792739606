// pgd_api.cu -- the C ABI of libpgd.so (declared in include/pgd.h): argument
// checks, grid planning, TMA descriptor encoding, workspace ownership and the
// launches.  No call here synchronises with the host except
// pgd_get_device_error() and workspace growth.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "pgd.h"
#include "pgd_grid.h"
#include "pgd_launch.h"

namespace {

using namespace pgd;

// Device flag word (bit set; see kFlag* in pgd_ptx.cuh).  Host code reaches it
// through cudaGetSymbolAddress, once per device.
__device__ uint32_t g_flags;

constexpr int kMaxDevices = 64;
constexpr int kMaxCtasPerSmForSizing = 4;

struct DeviceState {
    std::atomic<bool> init{false};   // set once, after the fields below
    int sms = 0;
    uint32_t *flags = nullptr;
    void *ws = nullptr;        // library-owned decode workspace (split partials)
    size_t ws_bytes = 0;
    int32_t *counters = nullptr;   // per-(sequence, KV head) arrival counters,
    size_t counter_cap = 0;        // zero between calls; grown on demand
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];

pgd_status cuda_fail(cudaError_t) { return PGD_ERR_CUDA; }

// The append kernels index a token's chunks with 32-bit integers.
constexpr int32_t kMaxAppendHeads = 65536;

pgd_status device_state(DeviceState **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PGD_ERR_CUDA;
    DeviceState &d = g_dev[dev];
    if (!d.init.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!d.init.load(std::memory_order_relaxed)) {
            if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
                return PGD_ERR_CUDA;
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_flags) != cudaSuccess) return PGD_ERR_CUDA;
            d.flags = static_cast<uint32_t *>(p);
            d.init.store(true, std::memory_order_release);
        }
    }
    *out = &d;
    return PGD_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over a KV cache [num_blocks][hkv][bs][D] viewed as 4-D
// (inner 128-byte line, token row, line within the row, block*hkv + head):
// one box = one (block, head) tile, landing in shared memory as
// [line][token][128 B] with the 128-byte swizzle.
pgd_status encode_kv_map(CUtensorMap *m, const void *base, int D, int E, int bs,
                         long long rows) {
    auto fn = encode_fn();
    if (!fn) return PGD_ERR_CUDA;
    const int lines = D * E / 128;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(128 / E), static_cast<cuuint64_t>(bs),
                          static_cast<cuuint64_t>(lines), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(D * E), 128,
                             static_cast<cuuint64_t>(bs) * D * E};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / E), static_cast<cuuint32_t>(bs),
                         static_cast<cuuint32_t>(lines), 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(m, E == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                    4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? PGD_OK : PGD_ERR_CUDA;
}

// Encoding a tensor map costs a driver call on the host, and a serving loop
// passes the same caches on every step, so each host thread keeps the maps it
// encoded last.  A map holds only the address, shape and strides it was
// encoded from, so an entry with the same key is the same map whatever
// happened to the memory in between.
struct KvMapKey {
    const void *base;
    long long rows;
    int D, E, bs;
    bool operator==(const KvMapKey &o) const {
        return base == o.base && rows == o.rows && D == o.D && E == o.E && bs == o.bs;
    }
};

pgd_status cached_kv_map(CUtensorMap *m, const void *base, int D, int E, int bs,
                         long long rows) {
    constexpr int kEntries = 8;
    struct Entry {
        KvMapKey key;
        CUtensorMap map;
        bool used;
    };
    thread_local Entry cache[kEntries] = {};
    thread_local int next = 0;
    const KvMapKey key{base, rows, D, E, bs};
    for (const Entry &e : cache)
        if (e.used && e.key == key) {
            *m = e.map;
            return PGD_OK;
        }
    const pgd_status st = encode_kv_map(m, base, D, E, bs, rows);
    if (st != PGD_OK) return st;
    Entry &e = cache[next];
    next = (next + 1) % kEntries;
    e.key = key;
    e.map = *m;
    e.used = true;
    return PGD_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
    size_t lse, opart, total;
};

// Caller or library workspace: split partials only (no zeroing needed).
WsLayout ws_layout(int g, int D, long long grid) {
    WsLayout w;
    w.lse = 0;
    w.opart = round256(sizeof(float) * 2 * grid * g);
    w.total = w.opart + round256(sizeof(float) * 2 * grid * g * D);
    return w;
}

// Library-owned arrival counters for `units` (sequence, KV head) pairs.
// Every completed launch leaves them zero; growth re-zeroes them.
pgd_status ensure_counters(DeviceState *d, long long units, cudaStream_t s) {
    std::lock_guard<std::mutex> lk(g_mu);
    if (d->counter_cap >= static_cast<size_t>(units)) return PGD_OK;
    if (d->counters) {
        cudaError_t e = cudaFree(d->counters);   // synchronises the device
        if (e != cudaSuccess) return cuda_fail(e);
        d->counters = nullptr;
        d->counter_cap = 0;
    }
    const size_t cap = std::max<size_t>(static_cast<size_t>(units), 4096);
    void *p = nullptr;
    cudaError_t e = cudaMalloc(&p, cap * sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaMemsetAsync(p, 0, cap * sizeof(int32_t), s);
    if (e != cudaSuccess) {
        cudaFree(p);
        return cuda_fail(e);
    }
    d->counters = static_cast<int32_t *>(p);
    d->counter_cap = cap;
    return PGD_OK;
}

using LaunchFn = cudaError_t (*)(const DecodeLaunchArgs &);
using OccFn = int (*)();

struct Variant {
    LaunchFn launch;
    OccFn occ;
};

template <int D, bool FP8>
bool pick_bs(int bs, int nt, Variant *v) {
#define PGD_CASE(BS, NT)                                                          \
    if (bs == BS && nt == NT) {                                                   \
        *v = {&launch_decode<D, BS, NT, FP8>, &decode_ctas_per_sm<D, BS, NT, FP8>}; \
        return true;                                                              \
    }
    PGD_CASE(16, 1) PGD_CASE(32, 1) PGD_CASE(64, 1)
    PGD_CASE(16, 2) PGD_CASE(32, 2) PGD_CASE(64, 2)
    PGD_CASE(16, 4) PGD_CASE(32, 4) PGD_CASE(64, 4)
#undef PGD_CASE
    return false;
}

// Consumer math of the decode kernels (pgd_set_decode_math); process-wide.
std::atomic<int> g_math{PGD_MATH_TENSOR_CORE};

// Limit of the decode kernels' pipeline waits in ns (pgd_debug_set_wait_limit_ns).
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};

template <int CC>
bool pick_cuda_core(int bs, Variant *v) {
    if (bs == 16) *v = {&launch_decode<128, 16, 1, false, CC>, &decode_ctas_per_sm<128, 16, 1, false, CC>};
    else if (bs == 32) *v = {&launch_decode<128, 32, 1, false, CC>, &decode_ctas_per_sm<128, 32, 1, false, CC>};
    else if (bs == 64) *v = {&launch_decode<128, 64, 1, false, CC>, &decode_ctas_per_sm<128, 64, 1, false, CC>};
    else return false;
    return true;
}

bool pick_variant(int D, int bs, int nt, bool fp8, int rows, Variant *v) {
    if (g_math.load() == PGD_MATH_CUDA_CORE) {
        if (fp8 || D != 128 || rows > 8) return false;
        return rows <= 4 ? pick_cuda_core<4>(bs, v) : pick_cuda_core<8>(bs, v);
    }
    if (!fp8 && D == 128) return pick_bs<128, false>(bs, nt, v);
    if (!fp8 && D == 256) return pick_bs<256, false>(bs, nt, v);
    if (fp8 && D == 128) return pick_bs<128, true>(bs, nt, v);
    return false;
}

bool supported_block(int bs) { return bs == 16 || bs == 32 || bs == 64; }
bool supported_group(int g) { return g >= 1 && g <= 16; }

}  // namespace

extern "C" {

const char *pgd_status_string(pgd_status s) {
    switch (s) {
        case PGD_OK: return "ok";
        case PGD_ERR_INVALID_ARG: return "invalid argument";
        case PGD_ERR_UNSUPPORTED: return "unsupported shape";
        case PGD_ERR_CUDA: return "CUDA error";
        case PGD_ERR_DEVICE_BOUNDS: return "device flagged an out-of-range index";
        case PGD_ERR_TIMEOUT: return "device flagged a pipeline wait timeout";
        case PGD_ERR_WORKSPACE: return "workspace too small";
    }
    return "unknown status";
}

const char *pgd_version(void) { return "0.1.0"; }

pgd_status pgd_kv_append(const void *k_new, const void *v_new, const int64_t *slot_mapping,
                         int32_t num_tokens, void *k_cache, void *v_cache, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int32_t num_blocks,
                         pgd_kv_dtype kv_dtype, void *stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PGD_ERR_INVALID_ARG;
    if (kv_dtype != PGD_KV_BF16 && kv_dtype != PGD_KV_FP8_E4M3) return PGD_ERR_INVALID_ARG;
    if (head_dim != 128 && head_dim != 256) return PGD_ERR_UNSUPPORTED;
    if (num_kv_heads > kMaxAppendHeads) return PGD_ERR_UNSUPPORTED;
    if (!supported_block(block_size)) return PGD_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PGD_OK;
    if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache) return PGD_ERR_INVALID_ARG;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) ||
        !aligned(v_cache, 16) || !aligned(slot_mapping, 8))
        return PGD_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    pgd_status st = device_state(&d);
    if (st != PGD_OK) return st;
    const int row_bytes = head_dim * (kv_dtype == PGD_KV_BF16 ? 2 : 1);
    cudaError_t e = launch_kv_append(k_new, v_new, slot_mapping, num_tokens, k_cache, v_cache,
                                     num_kv_heads, row_bytes, block_size,
                                     static_cast<int64_t>(num_blocks) * block_size, d->flags,
                                     static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PGD_OK : cuda_fail(e);
}

pgd_status pgd_kv_append_quant(const void *k_new, const void *v_new, const int64_t *slot_mapping,
                               int32_t num_tokens, void *k_cache, void *v_cache,
                               const float *k_scale, const float *v_scale, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int32_t num_blocks,
                               void *stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return PGD_ERR_INVALID_ARG;
    if (head_dim != 128 && head_dim != 256) return PGD_ERR_UNSUPPORTED;
    if (num_kv_heads > kMaxAppendHeads) return PGD_ERR_UNSUPPORTED;
    if (!supported_block(block_size)) return PGD_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PGD_OK;
    if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale)
        return PGD_ERR_INVALID_ARG;
    if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 8) ||
        !aligned(v_cache, 8) || !aligned(slot_mapping, 8) || !aligned(k_scale, 4) ||
        !aligned(v_scale, 4))
        return PGD_ERR_INVALID_ARG;
    DeviceState *d = nullptr;
    pgd_status st = device_state(&d);
    if (st != PGD_OK) return st;
    cudaError_t e = launch_kv_append_quant(k_new, v_new, slot_mapping, num_tokens, k_cache,
                                           v_cache, k_scale, v_scale, num_kv_heads, head_dim,
                                           block_size,
                                           static_cast<int64_t>(num_blocks) * block_size,
                                           d->flags, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PGD_OK : cuda_fail(e);
}

size_t pgd_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_q_heads % num_kv_heads)
        return 0;
    DeviceState *d = nullptr;
    if (device_state(&d) != PGD_OK) return 0;
    const long long grid = static_cast<long long>(d->sms) * kMaxCtasPerSmForSizing;
    return ws_layout(num_q_heads / num_kv_heads, head_dim, grid).total;
}

}  // extern "C"

namespace {

// Shared body of pgd_paged_decode_attention and pgd_decode_step (library
// or caller workspace; k_new / v_new non-null selects the fused append).
pgd_status decode_impl(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *block_table, int32_t max_blocks_per_seq,
                       const int32_t *context_lens, int32_t num_seqs, int32_t max_context_len,
                       int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                       int32_t block_size, int32_t num_blocks, float scale,
                       pgd_kv_dtype kv_dtype, const float *k_scale, const float *v_scale,
                       const void *k_new, const void *v_new, void *out, float *lse_out,
                       void *workspace, size_t workspace_bytes, int32_t num_ctas,
                       void *stream, int32_t q_len = 1, int32_t window = 0,
                       bool out_f32 = false) {
    // ---- host-side checks (nothing is enqueued on failure) ------------------
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || num_ctas < 0 || q_len < 1 ||
        window < 0)
        return PGD_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads) return PGD_ERR_INVALID_ARG;
    if (kv_dtype != PGD_KV_BF16 && kv_dtype != PGD_KV_FP8_E4M3) return PGD_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PGD_ERR_INVALID_ARG;
    const int g = num_q_heads / num_kv_heads;
    const bool fp8 = kv_dtype == PGD_KV_FP8_E4M3;
    if (!supported_group(g) || !supported_block(block_size)) return PGD_ERR_UNSUPPORTED;
    if (head_dim != 128 && head_dim != 256) return PGD_ERR_UNSUPPORTED;
    if (fp8 && head_dim != 128) return PGD_ERR_UNSUPPORTED;
    const int rows = g * q_len;                 // query rows per (sequence, KV head)
    if (rows > 32) return PGD_ERR_UNSUPPORTED;
    if (static_cast<long long>(num_blocks) * num_kv_heads >= INT_MAX ||
        static_cast<long long>(max_blocks_per_seq) * block_size >= INT_MAX)
        return PGD_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PGD_OK;
    if (!q || !k_cache || !v_cache || !block_table || !context_lens || !out)
        return PGD_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return PGD_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 16) || !aligned(out, 16) ||
        !aligned(block_table, 4) || !aligned(context_lens, 4) || (lse_out && !aligned(lse_out, 4)) ||
        (workspace && !aligned(workspace, 16)))
        return PGD_ERR_INVALID_ARG;
    if (!workspace && workspace_bytes) return PGD_ERR_INVALID_ARG;
    if ((k_new == nullptr) != (v_new == nullptr)) return PGD_ERR_INVALID_ARG;
    if (k_new && (!aligned(k_new, 16) || !aligned(v_new, 16))) return PGD_ERR_INVALID_ARG;
    if (k_new && q_len != 1) return PGD_ERR_UNSUPPORTED;   // fused append: one new token

    DeviceState *d = nullptr;
    pgd_status st = device_state(&d);
    if (st != PGD_OK) return st;
    const int nt = rows > 16 ? 4 : rows > 8 ? 2 : 1;   // n-tiles of 8 query rows
    Variant var;
    if (!pick_variant(head_dim, block_size, nt, fp8, rows, &var)) return PGD_ERR_UNSUPPORTED;

    // ---- grid: a full wave of resident CTAs, fewer for small batches ---------
    long long grid = num_ctas;
    if (grid == 0) {
        const int occ = var.occ();
        if (occ <= 0) return PGD_ERR_CUDA;
        grid = auto_grid(d->sms, occ, num_seqs, num_kv_heads, max_blocks_per_seq, block_size,
                         max_context_len, unit_cost_tiles(head_dim, block_size, fp8));
    }
    if (grid > (1LL << 24)) return PGD_ERR_INVALID_ARG;

    // ---- workspace --------------------------------------------------------------
    const WsLayout lay = ws_layout(rows, head_dim, grid);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = ensure_counters(d, static_cast<long long>(num_seqs) * num_kv_heads, s)) != PGD_OK)
        return st;
    if (!ws) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (d->ws_bytes < lay.total) {
            if (d->ws) {
                cudaError_t e = cudaFree(d->ws);   // synchronises the device
                if (e != cudaSuccess) return cuda_fail(e);
                d->ws = nullptr;
                d->ws_bytes = 0;
            }
            size_t want = std::max(lay.total, size_t(1) << 20);
            void *p = nullptr;
            cudaError_t e = cudaMalloc(&p, want);
            if (e != cudaSuccess) return cuda_fail(e);
            d->ws = p;
            d->ws_bytes = want;
        }
        ws = static_cast<uint8_t *>(d->ws);
    } else if (workspace_bytes < lay.total) {
        return PGD_ERR_WORKSPACE;
    }

    // ---- TMA descriptors and launch ------------------------------------------------
    DecodeLaunchArgs a;
    std::memset(&a, 0, sizeof(a));
    const int E = fp8 ? 1 : 2;
    const long long kv_rows = static_cast<long long>(num_blocks) * num_kv_heads;
    if ((st = cached_kv_map(&a.tmK, k_cache, head_dim, E, block_size, kv_rows)) != PGD_OK) return st;
    if ((st = cached_kv_map(&a.tmV, v_cache, head_dim, E, block_size, kv_rows)) != PGD_OK) return st;
    DecodeParams &p = a.p;
    p.q = static_cast<const uint16_t *>(q);
    p.out = static_cast<uint16_t *>(out);
    p.lse_out = lse_out;
    p.block_table = block_table;
    p.context_lens = context_lens;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.k_new = static_cast<const uint8_t *>(k_new);
    p.v_new = static_cast<const uint8_t *>(v_new);
    p.k_cache = static_cast<uint8_t *>(const_cast<void *>(k_cache));
    p.v_cache = static_cast<uint8_t *>(const_cast<void *>(v_cache));
    p.counters = d->counters;
    p.lse_part = reinterpret_cast<float *>(ws + lay.lse);
    p.o_part = reinterpret_cast<float *>(ws + lay.opart);
    p.flags = d->flags;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = g;
    p.num_blocks = num_blocks;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.unit_cost = unit_cost_tiles(head_dim, block_size, fp8);
    p.q_len = q_len;
    p.window = window;
    p.rows = rows;
    p.out_f32 = out_f32 ? 1 : 0;
    p.wait_ns = g_wait_ns.load();
    a.grid = static_cast<int>(grid);
    a.stream = s;
    cudaError_t e = var.launch(a);
    return e == cudaSuccess ? PGD_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

pgd_status pgd_paged_decode_attention(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
    int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale, void *out, float *lse_out, void *workspace,
    size_t workspace_bytes, int32_t num_ctas, void *stream) {
    return decode_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, context_lens,
                       num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                       block_size, num_blocks, scale, kv_dtype, k_scale, v_scale, nullptr,
                       nullptr, out, lse_out, workspace, workspace_bytes, num_ctas, stream);
}

pgd_status pgd_decode_step(
    const void *q, const void *k_new, const void *v_new, void *k_cache, void *v_cache,
    const int32_t *block_table, int32_t max_blocks_per_seq, const int32_t *context_lens,
    int32_t num_seqs, int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
    int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
    pgd_kv_dtype kv_dtype, const float *k_scale, const float *v_scale, void *out,
    float *lse_out, void *workspace, size_t workspace_bytes, int32_t num_ctas, void *stream) {
    if (num_seqs > 0 && (!k_new || !v_new)) return PGD_ERR_INVALID_ARG;
    return decode_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, context_lens,
                       num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                       block_size, num_blocks, scale, kv_dtype, k_scale, v_scale, k_new, v_new,
                       out, lse_out, workspace, workspace_bytes, num_ctas, stream);
}

pgd_status pgd_paged_decode_attention_ex(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
    int32_t max_context_len, int32_t q_len, int32_t window, int32_t num_q_heads,
    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
    pgd_kv_dtype kv_dtype, const float *k_scale, const float *v_scale, void *out,
    float *lse_out, void *workspace, size_t workspace_bytes, int32_t num_ctas, void *stream) {
    return decode_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, context_lens,
                       num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                       block_size, num_blocks, scale, kv_dtype, k_scale, v_scale, nullptr,
                       nullptr, out, lse_out, workspace, workspace_bytes, num_ctas, stream,
                       q_len, window);
}

pgd_status pgd_paged_decode_partial(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
    int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale, float *o_part, float *lse_part, void *workspace,
    size_t workspace_bytes, int32_t num_ctas, void *stream) {
    if (num_seqs > 0 && !lse_part) return PGD_ERR_INVALID_ARG;
    return decode_impl(q, k_cache, v_cache, block_table, max_blocks_per_seq, context_lens,
                       num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim,
                       block_size, num_blocks, scale, kv_dtype, k_scale, v_scale, nullptr,
                       nullptr, o_part, lse_part, workspace, workspace_bytes, num_ctas, stream,
                       1, 0, true);
}

pgd_status pgd_set_decode_math(pgd_decode_math math) {
    if (math != PGD_MATH_TENSOR_CORE && math != PGD_MATH_CUDA_CORE) return PGD_ERR_INVALID_ARG;
    g_math.store(math);
    return PGD_OK;
}

pgd_decode_math pgd_get_decode_math(void) {
    return static_cast<pgd_decode_math>(g_math.load());
}

pgd_status pgd_debug_set_wait_limit_ns(uint64_t limit_ns) {
    g_wait_ns.store(limit_ns == 0 ? kDefaultWaitNs : limit_ns);
    return PGD_OK;
}

uint64_t pgd_debug_get_wait_limit_ns(void) { return g_wait_ns.load(); }

int64_t pgd_decode_grid(int32_t sms, int32_t ctas_per_sm, int32_t num_seqs,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                        int32_t max_blocks_per_seq, int32_t max_context_len, int32_t fp8) {
    if (sms <= 0 || ctas_per_sm <= 0 || num_seqs < 0 || num_kv_heads <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || (fp8 != 0 && fp8 != 1) ||
        (head_dim != 128 && head_dim != 256) || !supported_block(block_size))
        return 0;
    return auto_grid(sms, ctas_per_sm, num_seqs, num_kv_heads, max_blocks_per_seq, block_size,
                     max_context_len, unit_cost_tiles(head_dim, block_size, fp8 != 0));
}

pgd_status pgd_kvp_plan(const int32_t *context_lens, int32_t num_seqs, int32_t block_size,
                        int32_t world_size, int32_t rank, int32_t *block_start,
                        int32_t *slice_len) {
    if (num_seqs < 0 || block_size <= 0 || world_size < 1 || rank < 0 || rank >= world_size)
        return PGD_ERR_INVALID_ARG;
    if (num_seqs == 0) return PGD_OK;
    if (!context_lens || !block_start || !slice_len) return PGD_ERR_INVALID_ARG;
    for (int32_t s = 0; s < num_seqs; ++s)
        if (context_lens[s] < 0) return PGD_ERR_INVALID_ARG;
    for (int32_t s = 0; s < num_seqs; ++s) {
        const long long n = context_lens[s];
        const long long nb = (n + block_size - 1) / block_size;
        const long long b0 = nb * rank / world_size, b1 = nb * (rank + 1) / world_size;
        const long long t0 = b0 * block_size, t1 = std::min(n, b1 * block_size);
        block_start[s] = static_cast<int32_t>(b0);
        slice_len[s] = static_cast<int32_t>(t1 > t0 ? t1 - t0 : 0);
    }
    return PGD_OK;
}

pgd_status pgd_merge_partials(const float *o_part, const float *lse_part, int32_t num_parts,
                              int32_t rows, int32_t head_dim, void *out, float *lse_out,
                              void *stream) {
    if (num_parts < 1 || rows < 0) return PGD_ERR_INVALID_ARG;
    if (head_dim != 128 && head_dim != 256) return PGD_ERR_UNSUPPORTED;
    if (rows == 0) return PGD_OK;
    if (!o_part || !lse_part || !out) return PGD_ERR_INVALID_ARG;
    if (!aligned(o_part, 16) || !aligned(lse_part, 4) || !aligned(out, 8) ||
        (lse_out && !aligned(lse_out, 4)))
        return PGD_ERR_INVALID_ARG;
    cudaError_t e = launch_merge_partials(o_part, lse_part, num_parts, rows, head_dim,
                                          static_cast<uint16_t *>(out), lse_out,
                                          static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? PGD_OK : cuda_fail(e);
}

pgd_status pgd_get_device_error(void *stream, uint32_t *flags) {
    DeviceState *d = nullptr;
    pgd_status st = device_state(&d);
    if (st != PGD_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t h = 0;
    if (cudaMemcpyAsync(&h, d->flags, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(d->flags, 0, sizeof(uint32_t), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return PGD_ERR_CUDA;
    if (flags) *flags = h;
    // a launch that bailed out may have left arrival counters behind
    if (h && d->counters &&
        (cudaMemsetAsync(d->counters, 0, d->counter_cap * sizeof(int32_t), s) != cudaSuccess ||
         cudaStreamSynchronize(s) != cudaSuccess))
        return PGD_ERR_CUDA;
    if (h & kFlagTimeout) return PGD_ERR_TIMEOUT;
    if (h) return PGD_ERR_DEVICE_BOUNDS;
    return PGD_OK;
}

pgd_status pgd_shutdown(void) {
    std::lock_guard<std::mutex> lk(g_mu);
    int cur = 0;
    cudaGetDevice(&cur);
    for (int i = 0; i < kMaxDevices; ++i) {
        if (g_dev[i].ws || g_dev[i].counters) {
            cudaSetDevice(i);
            cudaFree(g_dev[i].ws);
            cudaFree(g_dev[i].counters);
            g_dev[i].ws = nullptr;
            g_dev[i].ws_bytes = 0;
            g_dev[i].counters = nullptr;
            g_dev[i].counter_cap = 0;
        }
    }
    cudaSetDevice(cur);
    return PGD_OK;
}

pgd_status kv_append(const void *k_new, const void *v_new, const int64_t *slot_mapping,
                     int32_t num_tokens, void *k_cache, void *v_cache, int32_t num_kv_heads,
                     int32_t head_dim, int32_t block_size, int32_t num_blocks, void *stream) {
    return pgd_kv_append(k_new, v_new, slot_mapping, num_tokens, k_cache, v_cache, num_kv_heads,
                         head_dim, block_size, num_blocks, PGD_KV_BF16, stream);
}

pgd_status paged_decode_attention(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *block_table, int32_t max_blocks_per_seq,
                                  const int32_t *context_lens, int32_t num_seqs,
                                  int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t block_size, int32_t num_blocks, float scale, void *out,
                                  void *stream) {
    return pgd_paged_decode_attention(q, k_cache, v_cache, block_table, max_blocks_per_seq,
                                      context_lens, num_seqs, 0, num_q_heads, num_kv_heads,
                                      head_dim, block_size, num_blocks, scale, PGD_KV_BF16,
                                      nullptr, nullptr, out, nullptr, nullptr, 0, 0, stream);
}

}  // extern "C"

// ----------------------------------------------------------------------------
// Decode with no device allocation by the library.
//
// Some callers cannot let a library call cudaMalloc: a serving engine that
// reserves nearly all HBM for its KV-cache pool up front (a later cudaMalloc
// can fail, or push the pool out), a host whose policy is that every device
// byte goes through its own allocator and is accounted there, or a tight
// decode loop that cannot afford the device-wide synchronisation a cudaFree
// implies when a library buffer grows.  For them the scratch this kernel
// needs (split partials and the per-(sequence, KV head) arrival counters)
// lives in one fixed array of static device memory, below; each GPU that
// loads the library holds it until the process exits.
// ----------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(8) << 20;    // 8 MiB per device
constexpr long long kStaticMaxUnits = 65536;               // counters: 256 KiB
constexpr size_t kStaticCounterBytes = sizeof(int32_t) * kStaticMaxUnits;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct StaticScratch {
    std::atomic<bool> ready{false};   // set once, after ptr
    unsigned char *ptr = nullptr;   // device address of g_static_scratch
};
StaticScratch g_static[kMaxDevices];

// Resolve the device address of the static array for the current device.
// `g_static_scratch` in host code is only a stand-in symbol, so the address
// is looked up once per device (with that device current) and cached.
pgd_status static_scratch(unsigned char **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PGD_ERR_CUDA;
    StaticScratch &s = g_static[dev];
    if (!s.ready.load(std::memory_order_acquire)) {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!s.ready.load(std::memory_order_relaxed)) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return PGD_ERR_CUDA;
            s.ptr = static_cast<unsigned char *>(p);
            s.ready.store(true, std::memory_order_release);
        }
    }
    *out = s.ptr;
    return PGD_OK;
}

}  // namespace

extern "C" pgd_status pgd_paged_decode_attention_noalloc(
    const void *q, const void *k_cache, const void *v_cache, const int32_t *block_table,
    int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
    int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t block_size, int32_t num_blocks, float scale, pgd_kv_dtype kv_dtype,
    const float *k_scale, const float *v_scale, void *out, float *lse_out, int32_t num_ctas,
    void *stream) {
    // same host-side checks as pgd_paged_decode_attention
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || num_blocks <= 0 ||
        max_blocks_per_seq <= 0 || max_context_len < 0 || num_ctas < 0)
        return PGD_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads) return PGD_ERR_INVALID_ARG;
    if (kv_dtype != PGD_KV_BF16 && kv_dtype != PGD_KV_FP8_E4M3) return PGD_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PGD_ERR_INVALID_ARG;
    const int g = num_q_heads / num_kv_heads;
    const bool fp8 = kv_dtype == PGD_KV_FP8_E4M3;
    if (!supported_group(g) || !supported_block(block_size)) return PGD_ERR_UNSUPPORTED;
    if (head_dim != 128 && head_dim != 256) return PGD_ERR_UNSUPPORTED;
    if (fp8 && head_dim != 128) return PGD_ERR_UNSUPPORTED;
    if (static_cast<long long>(num_blocks) * num_kv_heads >= INT_MAX ||
        static_cast<long long>(max_blocks_per_seq) * block_size >= INT_MAX)
        return PGD_ERR_UNSUPPORTED;
    // the counters have a fixed capacity in the static array
    const long long units = static_cast<long long>(num_seqs) * num_kv_heads;
    if (units > kStaticMaxUnits) return PGD_ERR_WORKSPACE;
    if (num_seqs == 0) return PGD_OK;
    if (!q || !k_cache || !v_cache || !block_table || !context_lens || !out)
        return PGD_ERR_INVALID_ARG;
    if (fp8 && (!k_scale || !v_scale)) return PGD_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(q, 16) || !aligned(out, 16) ||
        !aligned(block_table, 4) || !aligned(context_lens, 4) || (lse_out && !aligned(lse_out, 4)))
        return PGD_ERR_INVALID_ARG;

    DeviceState *d = nullptr;
    pgd_status st = device_state(&d);
    if (st != PGD_OK) return st;
    unsigned char *scratch = nullptr;
    if ((st = static_scratch(&scratch)) != PGD_OK) return st;
    const int nt = g > 8 ? 2 : 1;
    Variant var;
    if (!pick_variant(head_dim, block_size, nt, fp8, g, &var)) return PGD_ERR_UNSUPPORTED;

    // grid: as the allocating entry point, capped so that the split partials
    // fit behind the counters in the static array.  A CTA's partials take
    // 8 * g * (head_dim + 1) bytes (two fp32 slots of g rows), so the array
    // holds the partials of at least 247 CTAs (g 16, head_dim 256) and of
    // 484 at head_dim 128: more than one wave of the automatic grid on a
    // 148-SM B200, where the cap never applies.
    const size_t avail = kStaticScratchBytes - kStaticCounterBytes;
    long long grid = num_ctas;
    if (grid == 0) {
        const int occ = var.occ();
        if (occ <= 0) return PGD_ERR_CUDA;
        grid = auto_grid(d->sms, occ, num_seqs, num_kv_heads, max_blocks_per_seq, block_size,
                         max_context_len, unit_cost_tiles(head_dim, block_size, fp8));
        const long long per_cta = 8LL * g * (head_dim + 1);
        const long long fit = std::max(1LL, static_cast<long long>(avail - 512) / per_cta);
        if (grid > fit) {
            grid = fit;
            if (units < grid && grid % units <= grid / 8) grid -= grid % units;
        }
    }
    if (grid > (1LL << 24)) return PGD_ERR_INVALID_ARG;
    const WsLayout lay = ws_layout(g, head_dim, grid);
    if (lay.total > avail) return PGD_ERR_WORKSPACE;   // an explicit num_ctas too large

    // the counters must start at zero; the partials need no clearing
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(int32_t) * units, s);
    if (e != cudaSuccess) return cuda_fail(e);

    DecodeLaunchArgs a;
    std::memset(&a, 0, sizeof(a));
    const int E = fp8 ? 1 : 2;
    const long long rows = static_cast<long long>(num_blocks) * num_kv_heads;
    if ((st = cached_kv_map(&a.tmK, k_cache, head_dim, E, block_size, rows)) != PGD_OK) return st;
    if ((st = cached_kv_map(&a.tmV, v_cache, head_dim, E, block_size, rows)) != PGD_OK) return st;
    uint8_t *parts = scratch + kStaticCounterBytes;
    DecodeParams &p = a.p;
    p.q = static_cast<const uint16_t *>(q);
    p.out = static_cast<uint16_t *>(out);
    p.lse_out = lse_out;
    p.block_table = block_table;
    p.context_lens = context_lens;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.counters = reinterpret_cast<int32_t *>(scratch);
    p.lse_part = reinterpret_cast<float *>(parts + lay.lse);
    p.o_part = reinterpret_cast<float *>(parts + lay.opart);
    p.flags = d->flags;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = g;
    p.num_blocks = num_blocks;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.unit_cost = unit_cost_tiles(head_dim, block_size, fp8);
    p.q_len = 1;
    p.window = 0;
    p.rows = g;
    p.wait_ns = g_wait_ns.load();
    a.grid = static_cast<int>(grid);
    a.stream = s;
    e = var.launch(a);
    return e == cudaSuccess ? PGD_OK : cuda_fail(e);
}
