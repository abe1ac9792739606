// pgd_decode.cuh -- split-KV paged GQA decode attention kernel for sm_100a.
//
// What it computes ("attention kernels", froggydisk: sections "standard
// attention", "FlashAttention", "prefill and decode attention", "paged KV and
// kernels"; "batching and attention", beengineer500, sections 2.4 and 3.4):
// for every sequence s and query head i (KV head h = i / g)
//     out[s][i] = softmax(scale * q[s][i] . K_t) . V_t  over t < context_lens[s],
// with K_t / V_t read through the block table, and lse[s][i] its log-sum-exp.
//
// Work decomposition.  The batch is flattened into tiles (s, h, j): KV head h
// of logical block j of sequence s, ordered by s, then h, then j; each
// (s, h) unit also weighs a fixed cost, so that a CTA given many short units
// gets fewer of them.  The total is cut into G equal contiguous ranges, one
// per CTA, so every CTA streams about the same KV bytes whatever the length
// mix ("prefill and decode attention": split along the KV length so that all
// SMs read at once).  Every CTA derives the cut from context_lens itself (no
// host round trip).  Inside its range a CTA walks "segments" (the part of one
// (s, h) unit that falls in the range).  A segment that covers its whole unit
// writes `out` directly; otherwise it writes a partial (o, lse) and the CTA
// that completes the unit's last share merges the partials by log-sum-exp.
//
// CTA = 4 consumer warps + 1 producer warp + 1 appender warp.  The producer
// is the only warp that reads the K/V inputs: it walks the segments, writes a
// descriptor for each into a small shared-memory ring together with the
// unit's query rows (bulk copy), loads the block-table entries 32 at a time
// (the next unit's while it issues the current one's tiles), and issues one
// TMA tensor load per (block, KV head) tile of K and of V into a ring of
// 64-token stages (128-byte swizzle, mbarrier completion).  Each K/V tile is
// fetched once and used by all g query heads of the group ("prefill and
// decode attention": GQA reuse).  In a fused decode step the appender warp
// writes each sequence's newest K/V row into the cache ahead of the producer
// ("batching and attention" 3.4: the new token's slot), so the append costs
// no extra launch.
//
// Consumer warp w owns tokens 16w .. 16w+15 of every stage and keeps its own
// online softmax ("FlashAttention") over them, with a small tensor-core
// contraction (mma.sync m16n8k16, fp32 accumulate) whose roles are
// transposed so that the unit's query rows are the narrow N = 8 dimension:
//   S^T[tokens][rows] = K[tokens][d] . Q^T[d][rows]
//   row max over the warp's tokens (shuffles) -> p = exp2(S - m)
//   P^T to the B-operand layout by a warp transpose (movmatrix)
//   O^T[d][rows] += V^T[d][tokens] . P^T[tokens][rows]  (all of D)
// The four warps' states are merged once per segment, in a fixed order.
// With bf16 K/V the weights p enter the PV product as two bf16 terms,
// p_hi = bf16(p) and p_lo = bf16(p - p_hi) (about 16 significant bits), and
// the normaliser sums the fp32 p; with FP8 K/V they enter as f16 (11 bits)
// and the normaliser sums those rounded values.  A row's reference max moves
// only when a score exceeds it by more than 2^8 (lazy rescaling).
#pragma once

#include "pgd_ptx.cuh"

namespace pgd {

struct DecodeParams {
    const uint16_t *q;            // bf16 bits [B][Hq][D], 16-byte aligned
    uint16_t *out;                // bf16 bits [B][Hq][D] (fp32 with out_f32)
    float *lse_out;               // [B][Hq] natural log, may be null
    const int32_t *block_table;   // [B][max_blocks_per_seq]
    const int32_t *context_lens;  // [B]
    const float *k_scale;         // [Hkv] (FP8 only)
    const float *v_scale;
    // fused append (decode step): the K/V rows of each sequence's newest
    // token, [B][Hkv][D] in the cache type, written to position ctx - 1
    // before that tile is read; null when the caller appended already.
    const uint8_t *k_new;
    const uint8_t *v_new;
    uint8_t *k_cache;             // raw cache pointers (fused append only)
    uint8_t *v_cache;
    int32_t *counters;            // [B * Hkv], zero between calls
    float *o_part;                // [2 * grid][rows][D]
    float *lse_part;              // [2 * grid][rows], log2 domain
    uint32_t *flags;              // device flag word
    int32_t max_blocks_per_seq;
    int32_t num_seqs, num_q_heads, num_kv_heads, group, num_blocks;
    float scale_log2;             // softmax scale * log2(e)
    int32_t unit_cost;            // work weight of a unit's fixed cost, in tiles
    // query rows per unit: q_len query tokens x group heads (rows <= 16).  q,
    // out are [B][q_len][Hq][D], lse [B][q_len][Hq]; query token i of a
    // sequence with n tokens sits at position n - q_len + i and sees tokens
    // below n - q_len + 1 + i, and with window > 0 only the last window of them.
    int32_t q_len, window, rows;
    // 1: out holds fp32 values (the unrounded split result a caller merges
    // with other splits of the same rows); 0: bf16
    int32_t out_f32;
    // limit of every pipeline wait in ns (kDefaultWaitNs unless a test of
    // the timeout path shortens it)
    uint64_t wait_ns;
};

constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 64;   // + producer warp + appender warp
constexpr int kAppSlots = 4;                // appender -> producer handoff ring
constexpr int kStageTokens = 16 * kConsumerWarps;
constexpr float kLn2 = 0.6931471805599453f;
// log2 of the largest softmax weight a consumer lets accumulate before it
// moves a row's reference max (lazy rescaling)
constexpr float kLazyRescale = 8.f;
constexpr uint32_t kBarConsumers = 1;

// Segment descriptor written by the producer, read by the consumers.
struct SegDesc {
    long long u;      // flattened index of the segment's first tile
    int s, h, j0, j1, n, ctx;
    int terminal;     // 1: no more segments for this CTA
    float ksc, vsc;   // FP8 per-KV-head scales (1 for bf16)
    int jlo;          // first block any query row of the unit sees
};

// CC = 0: tensor-core (mma.sync) consumers; CC = 4 or 8: the CUDA-core
// variant (FMA dot products with warp-shuffle reductions) for up to CC query
// rows, kept to compare the two on this bandwidth-bound path.
// NT = n-tiles of 8 query rows per unit: 1 (up to 8 rows), 2 (16) or 4 (32).
// With NT = 4 the consumer warps split into two row groups of 16 rows (warps
// 0, 1 and 2, 3) and each warp takes 32 tokens of every stage, so a stage is
// still read once for all 32 rows.
template <int D, int BS, int NT, bool FP8, int NSTAGES, int CC = 0>
struct DecodeCfg {
    static constexpr int E = FP8 ? 1 : 2;                // bytes per KV element
    static constexpr int ROW = D * E;                    // bytes per K/V row
    static constexpr int LINES = ROW / 128;              // 128-byte lines per row
    static constexpr int TILE = BS * ROW;                // one (block, head) tile
    static constexpr int BPS = kStageTokens / BS;        // blocks per stage
    static constexpr int STAGE_KV = BPS * TILE;          // K (or V) bytes per stage
    static constexpr int STAGE = 2 * STAGE_KV;
    static constexpr int RG = NT == 4 ? 2 : 1;           // row groups of consumer warps
    static constexpr int NTW = NT / RG;                  // n-tiles each warp holds
    static constexpr int GW = kConsumerWarps / RG;       // warps per row group
    static constexpr int SUBS = RG;                      // 16-token sub-tiles per warp and stage
    static constexpr int NP = 8 * NT;                    // padded query rows per unit
    static constexpr int DT = D / 16;                    // PV m-tiles (each warp: all of D)
    static constexpr int KSTEPS = D / 16;                // QK k-steps
    // head_dim 256 with tensor cores: the query rows stay in shared memory
    // for the whole segment (read by ldmatrix) instead of in registers
    static constexpr bool QSMEM = D == 256 && !FP8 && CC == 0;
    // The tensor-core consumers' query slot pads each row, so that the 8 rows
    // a fragment load touches fall in different banks: 16 bytes for bf16
    // (4-byte loads, and ldmatrix at head_dim 256), 32 bytes for FP8 (one
    // 8-byte load per k-step).  Each row then arrives by its own bulk copy.
    static constexpr bool QPAD = CC == 0;
    static constexpr int QROW = QPAD ? D * 2 + (FP8 ? 32 : 16) : D * 2;
    static constexpr int QSLOT = NP * QROW;              // query rows of one unit
    // descriptor ring depth (one slot for 16 or more query rows at head_dim
    // 128, so that two CTAs still fit on an SM; one for 32 rows at 256)
    static constexpr int NSEG =
        CC ? 2 : (NT == 4 ? 1 : (D == 128 ? (QSLOT >= 4096 ? 1 : 3) : 2));
    static constexpr int OROW = D + 4;                   // sO row stride in floats
    // shared memory carve-up (offsets from a 1024-aligned base)
    static constexpr int OFF_O = NSTAGES * STAGE;        // 8-row O merge buffers
    static constexpr int OBUF = 8 * OROW * 4;
    static constexpr int NOBUF = RG == 1 ? 2 : 1;        // A and B, or one per round
    static constexpr int OFF_Q = OFF_O + NOBUF * OBUF;
    static constexpr int OFF_SEG = OFF_Q + NSEG * QSLOT;
    static constexpr int OFF_RED = OFF_SEG + NSEG * (int)sizeof(SegDesc);   // warps' row max
    static constexpr int OFF_LSUM = OFF_RED + kConsumerWarps * NP * 4;      // warps' row sum
    static constexpr int OFF_ROW = OFF_LSUM + kConsumerWarps * NP * 4;      // rows' 1/L, lse
    // CUDA-core variant: each warp's softmax weights of a stage [16][CC] and
    // the rows' rescale factors [CC]
    static constexpr int PWF = 16 * 8 + 8;                // floats per warp
    static constexpr int OFF_PW = OFF_ROW + 2 * NP * 4;
    static constexpr int OFF_BAR = OFF_PW + (CC ? kConsumerWarps * PWF * 4 : 0);
    static constexpr int NBARS = 2 * NSTAGES + 2 * NSEG + 2 * kAppSlots;
    static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
    static constexpr int MISC_BYTES = 256;
    static constexpr int SMEM = OFF_MISC + MISC_BYTES + 1024;   // + alignment slack
    static_assert(ROW % 128 == 0, "rows must be whole 128-byte lines");
    static_assert(kStageTokens % BS == 0 && 32 % BPS == 0, "stage must hold whole blocks");
    static_assert(!FP8 || D == 128, "FP8 path is compiled for head_dim 128");
    static_assert(TILE % 1024 == 0, "tiles must keep the 1024-byte swizzle atom aligned");
    static_assert(sizeof(SegDesc) % 16 == 0, "descriptor alignment");
    static_assert(OFF_Q % 16 == 0, "bulk copies need 16-byte aligned destinations");
    static_assert(D != 128 || SMEM <= 113 * 1024, "two CTAs per SM at head_dim 128");
    static_assert(SMEM <= 227 * 1024, "shared memory of one CTA");
};

struct Misc {                 // CTA-wide scalars in shared memory
    long long pfx0;           // flattened index of the first tile of sequence s0
    int s0;
    int is_last;
    int found;
    int win_ok;               // win holds the context lengths of s0 .. s0 + 31
    long long warp_tmp[8];
    int win[32];
};

// ------------------------------------------------------------------ helpers
template <int BS>
__device__ __forceinline__ int ctx_of(const DecodeParams &p, int s) {
    int n = __ldg(p.context_lens + s);
    const int cap = p.max_blocks_per_seq * BS;
    if (n < 0 || n > cap) {
        raise_flag(p.flags, kFlagContextLen);
        n = n < 0 ? 0 : cap;
    }
    return n;
}

template <int BS>
__device__ __forceinline__ int nblk_of(int ctx) { return (ctx + BS - 1) / BS; }

// Block-wide sum over all kThreads threads (int64).
__device__ __forceinline__ long long block_sum(long long v, Misc *m) {
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5;
    __syncthreads();
    if ((threadIdx.x & 31) == 0) m->warp_tmp[w] = v;
    __syncthreads();
    long long t = 0;
    for (int i = 0; i < kThreads / 32; ++i) t += m->warp_tmp[i];
    __syncthreads();
    return t;
}

// Block-wide inclusive scan over kThreads threads (int64); also returns the
// block total.
__device__ __forceinline__ long long block_scan(long long v, long long &total, Misc *m) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    for (int o = 1; o < 32; o <<= 1) {
        long long n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    __syncthreads();
    if (lane == 31) m->warp_tmp[w] = v;
    __syncthreads();
    long long before = 0;
    total = 0;
    for (int i = 0; i < kThreads / 32; ++i) {
        if (i < w) before += m->warp_tmp[i];
        total += m->warp_tmp[i];
    }
    __syncthreads();
    return v + before;
}

// The CTA that holds work index x (ranges are [c*U/G, (c+1)*U/G), all
// non-empty since G <= U).
__device__ __forceinline__ long long cta_of(long long x, long long U, long long G) {
    return ((x + 1) * G - 1) / U;
}

// Work weight of one (sequence, KV head) unit of n tiles: its tiles plus a
// fixed cost, so that a CTA given many short units gets fewer of them.
__device__ __forceinline__ long long unit_weight(int n, int unit_cost) {
    return n > 0 ? (long long)n + unit_cost : 0;
}

// First block any query row of a unit with ctx tokens sees: the window of
// its first query token (position ctx - q_len) starts there; 0 without one.
template <int BS>
__device__ __forceinline__ int first_block(int ctx, const DecodeParams &p) {
    if (p.window <= 0) return 0;
    return max(0, ctx - p.q_len + 1 - p.window) / BS;
}

// Walk over the units of a CTA's work range (producer and appender; every
// lane of the warp walks in step).  Unit (s, h) reads blocks jlo .. n-1 and
// occupies work indices [a, a + w): its n - jlo tiles first, then the
// fixed-cost slots, which hold no tiles.  The context lengths of 32
// consecutive sequences sit one per lane (wbase, wval) and are read by
// shuffle, so the walk issues one coalesced load per 32 sequences instead of
// a dependent load per sequence.
struct Cursor {
    int s, h, n, ctx, jlo;
    long long a, w;
    int wbase, wval;
};

template <int BS>
__device__ __forceinline__ int window_ctx(Cursor &c, const DecodeParams &p, int s) {
    const int lane = threadIdx.x & 31;
    if (s < c.wbase || s >= c.wbase + 32) {
        c.wbase = s;
        c.wval = s + lane < p.num_seqs ? ctx_of<BS>(p, s + lane) : 0;
    }
    return __shfl_sync(0xffffffffu, c.wval, s - c.wbase);
}

template <int BS>
__device__ __forceinline__ void set_seq(Cursor &c, const DecodeParams &p) {
    c.ctx = window_ctx<BS>(c, p, c.s);
    c.n = nblk_of<BS>(c.ctx);
    c.jlo = first_block<BS>(c.ctx, p);
    c.w = unit_weight(c.n - c.jlo, p.unit_cost);
}

template <int BS>
__device__ __forceinline__ void next_unit(Cursor &c, const DecodeParams &p) {
    c.a += c.w;
    if (++c.h == p.num_kv_heads) {
        c.h = 0;
        for (++c.s; c.s < p.num_seqs; ++c.s) {
            set_seq<BS>(c, p);
            if (c.n) break;
        }
    }
}

template <int BS>
__device__ __forceinline__ Cursor first_unit(const DecodeParams &p, int s0, long long pfx0,
                                            long long u0, const int *win) {
    Cursor c;
    c.s = s0;
    if (win) {                       // the prologue's copy of s0 .. s0 + 31
        c.wbase = s0;
        c.wval = win[threadIdx.x & 31];
    } else {
        c.wbase = -64;               // empty window: the first read loads it
        c.wval = 0;
    }
    set_seq<BS>(c, p);
    c.h = (int)((u0 - pfx0) / c.w);
    c.a = pfx0 + (long long)c.h * c.w;
    return c;
}

// Work weight of sequence s per KV head (prologue sums and the locate scan).
template <int BS>
__device__ __forceinline__ long long seq_weight(const DecodeParams &p, int s) {
    const int ctx = ctx_of<BS>(p, s);
    const int n = nblk_of<BS>(ctx);
    return unit_weight(n - first_block<BS>(ctx, p), p.unit_cost);
}

__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}

__device__ __forceinline__ long long lds64(uint32_t a) {
    long long v;
    asm volatile("ld.shared.b64 %0, [%1];" : "=l"(v) : "r"(a));
    return v;
}

// Log-sum-exp merge of one unit's split partials by the 128 consumer threads
// ("attention kernels", "prefill and decode attention"): with lse_c in the
// log2 domain, M = max_c lse_c, w_c = 2^(lse_c - M), out = sum w_c o_c / sum w_c.
// Each thread owns one query row and a strided set of float4 columns (in two
// passes when a unit has 32 rows); the weights are formed once per row and
// pass, and the partial rows are read several pieces at a time so that the L2
// round trips overlap.
template <int D>
__device__ __forceinline__ void merge_unit(const DecodeParams &p, long long ua, long long U,
                                           long long G, long long c_first, long long c_last,
                                           int s, int h) {
    constexpr int V4 = D / 4;                      // float4 columns per row
    constexpr int MAXC = (V4 + 7) / 8;             // columns per thread and pass
    const int R = p.rows, g = p.group;
    const int tph = kConsumers / R;                // threads per query row (R <= 32)
    const int head = threadIdx.x / tph, sub = threadIdx.x % tph;   // head: the query row
    if (head >= R) return;                         // 128 / R need not be exact
    // output row of query row `head`: query token head / g, head h*g + head % g
    const long long orow =
        ((long long)s * p.q_len + head / g) * p.num_q_heads + (long long)h * g + head % g;
    auto slot_of = [&](long long c) { return 2 * c + ((ua <= c * U / G) ? 0 : 1); };
    // One pass over the pieces in order, NG at a time with all their loads in
    // flight: running max M, weight sum W and weighted sum acc, rescaled
    // whenever M grows (the online softmax merge).
    constexpr int NG = D == 128 ? 4 : 2;
    float M = -INFINITY, W = 0.f;
    for (int cb = 0; cb < V4; cb += MAXC * tph) {
        M = -INFINITY;
        W = 0.f;
        float4 acc[MAXC];
#pragma unroll
        for (int i = 0; i < MAXC; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (long long c = c_first; c <= c_last; c += NG) {
            float l[NG];
            float4 v[NG][MAXC];
#pragma unroll
            for (int k = 0; k < NG; ++k) {
                const bool live = c + k <= c_last;
                const long long sl = slot_of(live ? c + k : c);
                l[k] = live ? __ldcg(p.lse_part + sl * R + head) : -INFINITY;
                const float4 *row =
                    reinterpret_cast<const float4 *>(p.o_part + (sl * R + head) * D);
#pragma unroll
                for (int i = 0; i < MAXC; ++i) {
                    const int col = cb + sub + i * tph;
                    v[k][i] = (live && col < V4) ? __ldcg(row + col)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
            float gm = M;
#pragma unroll
            for (int k = 0; k < NG; ++k) gm = fmaxf(gm, l[k]);
            const float Mu = gm == -INFINITY ? 0.f : gm;
            const float so = ex2(M - Mu);
            W *= so;
#pragma unroll
            for (int i = 0; i < MAXC; ++i) {
                acc[i].x *= so; acc[i].y *= so; acc[i].z *= so; acc[i].w *= so;
            }
#pragma unroll
            for (int k = 0; k < NG; ++k) {
                const float w = ex2(l[k] - Mu);
                W += w;
#pragma unroll
                for (int i = 0; i < MAXC; ++i) {
                    acc[i].x += w * v[k][i].x; acc[i].y += w * v[k][i].y;
                    acc[i].z += w * v[k][i].z; acc[i].w += w * v[k][i].w;
                }
            }
            M = gm;
        }
        const float inv = W > 0.f ? 1.f / W : 0.f;
#pragma unroll
        for (int i = 0; i < MAXC; ++i) {
            const int col = cb + sub + i * tph;
            if (col < V4) {
                if (p.out_f32) {
                    const float4 v = make_float4(acc[i].x * inv, acc[i].y * inv, acc[i].z * inv,
                                                 acc[i].w * inv);
                    *reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + orow * D +
                                                4 * col) = v;
                } else {
                    uint2 packed;
                    packed.x = pack_bf16x2(acc[i].x * inv, acc[i].y * inv);
                    packed.y = pack_bf16x2(acc[i].z * inv, acc[i].w * inv);
                    *reinterpret_cast<uint2 *>(p.out + orow * D + 4 * col) = packed;
                }
            }
        }
    }
    // every pass saw the same weights, so M and W are those of any pass
    if (p.lse_out && sub == 0)
        p.lse_out[orow] = W > 0.f ? (M + log2f(W)) * kLn2 : -INFINITY;
}

// ------------------------------------------------------------------ kernel
template <int D, int BS, int NT, bool FP8, int NSTAGES, int CC = 0>
__global__ void __launch_bounds__(kThreads, D == 128 ? 2 : 1)
paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const DecodeParams p) {
    using C = DecodeCfg<D, BS, NT, FP8, NSTAGES, CC>;
    static_assert(CC == 0 || (D == 128 && !FP8 && NT == 1 && (CC == 4 || CC == 8)),
                  "CUDA-core variant: bf16, head_dim 128, 4 or 8 rows");
    static_assert(sizeof(Misc) <= C::MISC_BYTES, "CTA scalars");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    Misc *misc = reinterpret_cast<Misc *>(smem + C::OFF_MISC);
    float *red = reinterpret_cast<float *>(smem + C::OFF_RED);
    float *lsum = reinterpret_cast<float *>(smem + C::OFF_LSUM);
    SegDesc *segs = reinterpret_cast<SegDesc *>(smem + C::OFF_SEG);
    const uint32_t sSeg = sbase + C::OFF_SEG;
    const uint32_t bar_full = sbase + C::OFF_BAR;
    const uint32_t bar_empty = bar_full + NSTAGES * 8;
    const uint32_t seg_full = bar_empty + NSTAGES * 8;
    const uint32_t seg_empty = seg_full + C::NSEG * 8;
    const uint32_t app_done = seg_empty + C::NSEG * 8;
    const uint32_t app_free = app_done + kAppSlots * 8;
    const uint32_t sO = sbase + C::OFF_O;
    float *rowinv = reinterpret_cast<float *>(smem + C::OFF_ROW);
    float *rowlse = rowinv + C::NP;
    const uint32_t sQ = sbase + C::OFF_Q;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.num_seqs, Hkv = p.num_kv_heads, g = p.group;
    const long long cta = blockIdx.x;

    // Programmatic dependent launch: let the next launch on the stream be
    // scheduled now, and wait until the previous one has completed and its
    // writes are visible before this grid reads anything from global memory.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (tid == 0) {
        for (int i = 0; i < NSTAGES; ++i) {
            mbar_init(bar_full + 8 * i, 1);
            mbar_init(bar_empty + 8 * i, kConsumerWarps);
        }
        for (int i = 0; i < C::NSEG; ++i) {
            mbar_init(seg_full + 8 * i, 1);
            mbar_init(seg_empty + 8 * i, kConsumerWarps);
        }
        for (int i = 0; i < kAppSlots; ++i) {
            mbar_init(app_done + 8 * i, 1);
            mbar_init(app_free + 8 * i, 1);
        }
        fence_mbar_init();
        misc->found = 0;
    }
    if (warp == kConsumerWarps && lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }

    // units with an empty context: out = 0, lse = -inf for all their query
    // rows.  Warp w of nw takes units w, w + nw, ...; its lanes write each
    // empty unit's q_len runs of g rows in 16-byte pieces.
    auto zero_fill = [&](long long w, long long nw) {
        const int ln = tid & 31;
        const int pieces = g * D * (p.out_f32 ? 4 : 2) / 16;   // of g rows
        for (long long v = w; v < (long long)B * Hkv; v += nw) {
            const int s = (int)(v / Hkv), h = (int)(v % Hkv);
            if (ctx_of<BS>(p, s) != 0) continue;   // the same length in every lane
            for (int i = 0; i < p.q_len; ++i) {
                const long long row0 =
                    ((long long)s * p.q_len + i) * p.num_q_heads + (long long)h * g;
                uint4 *o = reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(p.out) +
                                                     row0 * D * (p.out_f32 ? 4 : 2));
                for (int c = ln; c < pieces; c += 32) o[c] = make_uint4(0u, 0u, 0u, 0u);
                if (p.lse_out)
                    for (int e = ln; e < g; e += 32) p.lse_out[row0 + e] = -INFINITY;
            }
        }
    };

    // ---- prologue: total work and this CTA's range --------------------
    // Thread t reads the context lengths of sequences t*KS .. t*KS + KS - 1
    // of the first CH once and keeps them; one block scan gives every
    // sequence's work prefix.  Longer batches are summed in further passes.
    constexpr int KS = 4, CH = KS * kThreads;
    int cl[KS];
    long long wk[KS], tsum = 0;
#pragma unroll
    for (int k = 0; k < KS; ++k) {
        const int s = tid * KS + k;
        cl[k] = s < B ? ctx_of<BS>(p, s) : 0;
        wk[k] = s < B ? unit_weight(nblk_of<BS>(cl[k]) - first_block<BS>(cl[k], p), p.unit_cost)
                      : 0;
        tsum += wk[k];
    }
    long long W0;                                   // one KV head's work in the first CH
    const long long excl0 = block_scan(tsum, W0, misc) - tsum;
    long long U1 = W0;                              // one KV head's work in the batch
    for (int base = CH; base < B; base += kThreads) {
        const int s = base + tid;
        U1 += block_sum(s < B ? seq_weight<BS>(p, s) : 0, misc);
    }
    const long long U = U1 * Hkv;
    // CTAs beyond the work count get no range, so every range is non-empty
    const long long G = min((long long)gridDim.x, U);
    const long long u0 = cta < G ? cta * U / G : 0, u1 = cta < G ? (cta + 1) * U / G : 0;
    if (U == 0) {             // every context is empty
        zero_fill(cta * (kThreads / 32) + (tid >> 5), (long long)gridDim.x * (kThreads / 32));
        return;
    }
    if (u0 >= u1) return;   // nothing in flight, no barrier shared past this point

    // locate the sequence that holds work index u0
    {
        long long a = excl0 * Hkv;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int s = tid * KS + k;
            const long long w = wk[k] * Hkv;
            if (s < B && w > 0 && a <= u0 && u0 < a + w) {
                misc->s0 = s;
                misc->pfx0 = a;
                misc->found = 1;
            }
            a += w;
        }
    }
    __syncthreads();
    if (!misc->found) {       // u0 lies past the first CH sequences
        long long base = W0 * Hkv;
        for (int sb = CH; sb < B; sb += kThreads) {
            const int s = sb + tid;
            const long long wgt = s < B ? seq_weight<BS>(p, s) * Hkv : 0;
            long long tot;
            const long long incl = block_scan(wgt, tot, misc);
            const long long excl = base + incl - wgt;
            if (s < B && wgt > 0 && excl <= u0 && u0 < excl + wgt) {
                misc->s0 = s;
                misc->pfx0 = excl;
                misc->found = 1;
            }
            base += tot;
            __syncthreads();
            if (misc->found) break;
        }
    }
    // context lengths of s0 .. s0 + 31 for the walkers' first window
    {
        const int s0 = misc->s0;
#pragma unroll
        for (int k = 0; k < KS; ++k) {
            const int s = tid * KS + k;
            if (s >= s0 && s < s0 + 32) misc->win[s - s0] = cl[k];
        }
        if (tid == 0) misc->win_ok = (s0 + 32 <= CH || B <= CH) ? 1 : 0;
    }
    __syncthreads();
    const int *win0 = misc->win_ok ? misc->win : nullptr;

    if (warp == kConsumerWarps + 1) {
        // ================= appender warp (fused append only) ===============
        // Walks the same segments as the producer.  For each segment that
        // holds its unit's last block it writes the newest token's K and V
        // rows into the cache (position ctx - 1), orders those generic writes
        // before async-proxy reads, and signals the producer, which waits for
        // the signal before loading that block.  Only this CTA reads the
        // unit's last tile, so no other CTA can see the row half-written.
        // First it writes the empty units (one appender warp in each of the
        // G CTAs that have work).
        zero_fill(cta, G);
        if (p.k_new == nullptr) return;
        Cursor cur = first_unit<BS>(p, misc->s0, misc->pfx0, u0, win0);
        uint32_t ait = 0;
        for (; cur.a < u1; next_unit<BS>(cur, p)) {
            const long long r0 = max(0LL, u0 - cur.a);
            const long long r1 = min((long long)(cur.n - cur.jlo), u1 - cur.a);
            if (r0 < r1 && cur.jlo + r1 == cur.n) {
                const uint32_t as = ait % kAppSlots;
                bool ok = true;
                if (lane == 0 && ait >= (uint32_t)kAppSlots)
                    ok = mbar_wait_bounded(app_free + 8 * as, ((ait / kAppSlots) - 1) & 1, p.wait_ns);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) {
                    if (lane == 0) raise_flag(p.flags, kFlagTimeout);
                    return;
                }
                int pb = __ldg(p.block_table + (long long)cur.s * p.max_blocks_per_seq + cur.n - 1);
                if (pb < 0 || pb >= p.num_blocks) {
                    if (lane == 0) raise_flag(p.flags, kFlagBlockId);
                    pb = 0;
                }
                const long long dst =
                    (((long long)pb * Hkv + cur.h) * BS + (cur.ctx - 1) % BS) * C::ROW;
                const long long src = ((long long)cur.s * Hkv + cur.h) * C::ROW;
                constexpr int CH = C::ROW / 16;   // 16-byte chunks per row
                for (int c = lane; c < 2 * CH; c += 32) {
                    const bool isk = c < CH;
                    const int off = 16 * (isk ? c : c - CH);
                    const uint4 v =
                        __ldg(reinterpret_cast<const uint4 *>((isk ? p.k_new : p.v_new) + src + off));
                    *reinterpret_cast<uint4 *>((isk ? p.k_cache : p.v_cache) + dst + off) = v;
                }
                asm volatile("fence.proxy.async.global;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(app_done + 8 * as);
                ++ait;
            }
        }
        return;
    }

    if (warp == kConsumerWarps) {
        // ================= producer warp ====================================
        Cursor cur = first_unit<BS>(p, misc->s0, misc->pfx0, u0, win0);
        const uint32_t qtok = (uint32_t)(g * D * 2);          // one query token's rows
        uint32_t it = 0, sit = 0, ait = 0;
        bool ok = true;
        // FP8 scales of the first 32 KV heads, one per lane
        float ks_l = 1.f, vs_l = 1.f;
        if (FP8 && lane < Hkv) {
            ks_l = __ldg(p.k_scale + lane);
            vs_l = __ldg(p.v_scale + lane);
        }
        // the segment's blocks [j0, j1) of unit c (empty: only fixed-cost slots)
        auto seg_of = [&](const Cursor &c, int &j0, int &j1) {
            j0 = c.jlo + (int)max(0LL, u0 - c.a);
            j1 = c.jlo + (int)min((long long)(c.n - c.jlo), u1 - c.a);
        };
        // block ids of a segment's first 32 blocks, one per lane; the next
        // unit's are loaded while this unit's tiles are issued, so the walk
        // never waits on a dependent block-table load
        auto first_ids = [&](const Cursor &c, int j0, int j1) -> int {
            const int32_t *bt = p.block_table + (long long)c.s * p.max_blocks_per_seq;
            return j0 + lane < j1 ? __ldg(bt + j0 + lane) : 0;
        };
        // The units of one sequence (its KV heads) share its block-table row,
        // so a unit whose segment starts at the same block reuses the ids the
        // previous unit loaded, and the next sequence's ids are loaded as soon
        // as the walk enters a sequence: a whole sequence of units ahead.  A
        // walk of many short units then never waits on a block-table load.
        Cursor la = cur;             // first unit of the sequence after cur's
        int pf_la = 0, la_j0 = -1;
        auto look_ahead = [&](const Cursor &from) {
            la = from;
            while (la.a < u1 && la.s == from.s) next_unit<BS>(la, p);
            la_j0 = -1;
            if (la.a < u1) {
                int b0, b1;
                seg_of(la, b0, b1);
                pf_la = first_ids(la, b0, b1);
                la_j0 = b0;
            }
        };
        int pf = 0;
        if (cur.a < u1) {
            int a0, a1;
            seg_of(cur, a0, a1);
            pf = first_ids(cur, a0, a1);
            look_ahead(cur);
        }
        for (; cur.a < u1 && ok;) {
            int j0, j1;                                  // absolute blocks
            seg_of(cur, j0, j1);
            Cursor nxt = cur;
            next_unit<BS>(nxt, p);
            int pf_next = 0;
            if (nxt.a < u1) {
                int b0, b1;
                seg_of(nxt, b0, b1);
                if (nxt.s == cur.s && b0 == j0) {
                    pf_next = pf;                        // same row, same first block
                } else if (nxt.s == la.s && b0 == la_j0) {
                    pf_next = pf_la;                     // loaded a sequence ago
                    look_ahead(nxt);
                } else {
                    pf_next = first_ids(nxt, b0, b1);
                    look_ahead(nxt);
                }
            }
            if (j0 >= j1) {          // the range holds only this unit's fixed-cost slots
                cur = nxt;
                pf = pf_next;
                continue;
            }
            const int r0 = j0 - cur.jlo;
            float ksc = 1.f, vsc = 1.f;
            if (FP8) {
                ksc = __shfl_sync(0xffffffffu, ks_l, cur.h & 31);
                vsc = __shfl_sync(0xffffffffu, vs_l, cur.h & 31);
                if (cur.h >= 32) {
                    ksc = __ldg(p.k_scale + cur.h);
                    vsc = __ldg(p.v_scale + cur.h);
                }
            }
            // -- descriptor and query rows of the segment
            {
                const uint32_t slot = sit % C::NSEG;
                if (lane == 0 && sit >= (uint32_t)C::NSEG)
                    ok = mbar_wait_bounded(seg_empty + 8 * slot, ((sit / C::NSEG) - 1) & 1, p.wait_ns);
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
                if (lane == 0) {
                    SegDesc &d = segs[slot];
                    d.u = cur.a + r0;
                    d.s = cur.s;
                    d.h = cur.h;
                    d.j0 = j0;
                    d.j1 = j1;
                    d.n = cur.n;
                    d.ctx = cur.ctx;
                    d.terminal = 0;
                    d.ksc = ksc;
                    d.vsc = vsc;
                    d.jlo = cur.jlo;
                    const uint32_t bar = seg_full + 8 * slot;
                    mbar_arrive_expect_tx(bar, qtok * p.q_len);
                    // query rows: q_len runs of g contiguous heads, row = i*g + head
                    if (!C::QPAD)
                        for (int i = 0; i < p.q_len; ++i)
                            bulk_copy_g2s(sQ + slot * C::QSLOT + i * qtok,
                                          p.q + (((long long)cur.s * p.q_len + i) * p.num_q_heads +
                                                 (long long)cur.h * g) * D,
                                          qtok, bar);
                }
                if (C::QPAD) {
                    // one copy per row into the padded slot (after the expect-tx)
                    __syncwarp();
                    for (int r = lane; r < g * p.q_len; r += 32)
                        bulk_copy_g2s(sQ + slot * C::QSLOT + r * C::QROW,
                                      p.q + (((long long)cur.s * p.q_len + r / g) * p.num_q_heads +
                                             (long long)cur.h * g + r % g) * D,
                                      D * 2, seg_full + 8 * slot);
                }
                ++sit;
            }
            // a segment that holds its unit's last block takes the appended
            // row from the appender warp before that block is loaded
            const bool app_seg = p.k_new != nullptr && j1 == cur.n;
            // -- K/V tiles, block ids fetched 32 at a time (one chunk ahead)
            const int32_t *bt = p.block_table + (long long)cur.s * p.max_blocks_per_seq;
            int jc = j0;
            int pb_next = pf;
            while (jc < j1 && ok) {
                const int pb_cur = pb_next;
                const int jn = jc + 32;
                pb_next = jn + lane < j1 ? __ldg(bt + jn + lane) : 0;
                const int chunk_end = min(j1, jn);
                for (int jj = jc; jj < chunk_end; jj += C::BPS) {
                    const int nb = min(C::BPS, j1 - jj);
                    const uint32_t slot = it % NSTAGES;
                    if (lane == 0 && it >= (uint32_t)NSTAGES)
                        ok = mbar_wait_bounded(bar_empty + 8 * slot, ((it / NSTAGES) - 1) & 1, p.wait_ns);
                    if (app_seg && jj + nb == j1 && lane == 0 && ok) {
                        // the appended row is in this stage: wait for its write
                        const uint32_t as = ait % kAppSlots;
                        ok = mbar_wait_bounded(app_done + 8 * as, (ait / kAppSlots) & 1, p.wait_ns);
                        mbar_arrive(app_free + 8 * as);
                        ++ait;
                    }
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) break;
                    const uint32_t full = bar_full + 8 * slot;
                    if (lane == 0) mbar_arrive_expect_tx(full, (uint32_t)(nb * 2 * C::TILE));
                    const uint32_t dK = sbase + slot * C::STAGE, dV = dK + C::STAGE_KV;
#pragma unroll
                    for (int b = 0; b < C::BPS; ++b) {
                        int pb = __shfl_sync(0xffffffffu, pb_cur, (jj - jc + b) & 31);
                        if (b < nb && lane == 0) {
                            if (pb < 0 || pb >= p.num_blocks) {
                                raise_flag(p.flags, kFlagBlockId);
                                pb = 0;
                            }
                            const int32_t row = pb * Hkv + cur.h;
                            tma_load_4d(dK + b * C::TILE, &tmK, full, 0, 0, 0, row);
                            tma_load_4d(dV + b * C::TILE, &tmV, full, 0, 0, 0, row);
                        }
                    }
                    ++it;
                }
                jc = jn;
            }
            cur = nxt;
            pf = pf_next;
        }
        if (!ok && lane == 0) raise_flag(p.flags, kFlagTimeout);
        if (lane == 0) {
            // the terminal descriptor needs the slot of segment sit - NSEG back
            const uint32_t slot = sit % C::NSEG;
            bool free_slot = true;
            if (sit >= (uint32_t)C::NSEG)
                free_slot = mbar_wait_bounded(seg_empty + 8 * slot, ((sit / C::NSEG) - 1) & 1,
                                              p.wait_ns);
            // drain: every issued copy must land before the CTA may exit.  Each
            // slot waited on here has no later arrival, so its parity is exact;
            // segment sit - NSEG is skipped once the consumers released its
            // slot (they had read its query rows, so that copy had landed).
            const uint32_t first = it > NSTAGES ? it - NSTAGES : 0;
            for (uint32_t k = first; k < it; ++k)
                if (!mbar_wait_bounded(bar_full + 8 * (k % NSTAGES), (k / NSTAGES) & 1,
                                       kDrainWaitNs))
                    raise_flag(p.flags, kFlagTimeout);
            uint32_t qfirst = sit > C::NSEG ? sit - C::NSEG : 0;
            if (free_slot && sit >= (uint32_t)C::NSEG) qfirst = sit - C::NSEG + 1;
            for (uint32_t k = qfirst; k < sit; ++k)
                if (!mbar_wait_bounded(seg_full + 8 * (k % C::NSEG), (k / C::NSEG) & 1,
                                       kDrainWaitNs))
                    raise_flag(p.flags, kFlagTimeout);
            // terminal descriptor (also after a timeout, so that the consumers stop)
            if (free_slot) {
                segs[slot].terminal = 1;
                mbar_arrive(seg_full + 8 * slot);
            }
        }
        return;
    }

    // ==================== consumers (warps 0..3) ===========================
    const int gid = lane >> 2, t4 = lane & 3;
    uint32_t it = 0, sit = 0;

    for (;;) {
        // ---- next segment: descriptor + query fragments from shared memory
        const uint32_t qs = sit % C::NSEG;
        const bool seg_ok = mbar_wait_bounded(seg_full + 8 * qs, (sit / C::NSEG) & 1, p.wait_ns);
        if (!seg_ok) raise_flag(p.flags, kFlagTimeout);
        const uint32_t da = sSeg + qs * (uint32_t)sizeof(SegDesc);
        const long long useg = lds64(da + offsetof(SegDesc, u));
        const int s = (int)lds32(da + offsetof(SegDesc, s));
        const int h = (int)lds32(da + offsetof(SegDesc, h));
        const int j0 = (int)lds32(da + offsetof(SegDesc, j0));
        const int j1 = (int)lds32(da + offsetof(SegDesc, j1));
        const int nunit = (int)lds32(da + offsetof(SegDesc, n));
        const int ctx = (int)lds32(da + offsetof(SegDesc, ctx));
        const int terminal = (int)lds32(da + offsetof(SegDesc, terminal));
        const float ksc = __uint_as_float(lds32(da + offsetof(SegDesc, ksc)));
        const float vsc = __uint_as_float(lds32(da + offsetof(SegDesc, vsc)));
        const int jlo = (int)lds32(da + offsetof(SegDesc, jlo));
        // all consumers agree on leaving (a terminal descriptor, or a wait that
        // timed out, whose descriptor may be stale)
        if (named_bar_sync_or(kBarConsumers, kConsumers, !seg_ok || terminal)) return;
        const bool whole = (j0 == jlo && j1 == nunit);
        const int R = p.rows;

        float sl2 = p.scale_log2 * ksc;
        // output row of query row r: query token r / g, head h*g + r % g
        auto orow = [&](int r) -> long long {
            return ((long long)s * p.q_len + r / g) * p.num_q_heads + (long long)h * g + r % g;
        };
        // partial results: slot 2c for the CTA's first segment, 2c+1 for its last
        const long long pslot = 2 * cta + (useg == u0 ? 0 : 1);
        constexpr int CPR = D / 8;   // 8-float chunks per row
        // (A + B) / L (two merge buffers) or A / L (one) for rows r0 .. r0 + 7,
        // 8 consecutive dims per step: the output, or this CTA's partial result
        auto finalize_rows = [&](int r0) {
            for (int c = tid; c < 8 * CPR; c += kConsumers) {
                const int rl = c / CPR, d0 = (c % CPR) * 8, r = r0 + rl;
                if (r >= R) continue;
                const uint32_t a = sO + (rl * C::OROW + d0) * 4;
                uint32_t x[8], y[8];
                lds128(a, x[0], x[1], x[2], x[3]);
                lds128(a + 16, x[4], x[5], x[6], x[7]);
                if constexpr (C::NOBUF == 2) {
                    lds128(a + C::OBUF, y[0], y[1], y[2], y[3]);
                    lds128(a + C::OBUF + 16, y[4], y[5], y[6], y[7]);
                }
                const float inv = rowinv[r];
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    v[i] = __uint_as_float(x[i]);
                    if constexpr (C::NOBUF == 2) v[i] += __uint_as_float(y[i]);
                    v[i] *= inv;
                }
                if (whole) {
                    const long long at = orow(r) * D + d0;
                    if (p.out_f32) {
                        float4 *dst = reinterpret_cast<float4 *>(reinterpret_cast<float *>(p.out) + at);
                        dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                        dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    } else {
                        uint4 pk;
                        pk.x = pack_bf16x2(v[0], v[1]);
                        pk.y = pack_bf16x2(v[2], v[3]);
                        pk.z = pack_bf16x2(v[4], v[5]);
                        pk.w = pack_bf16x2(v[6], v[7]);
                        *reinterpret_cast<uint4 *>(p.out + at) = pk;
                    }
                    if (p.lse_out && d0 == 0) p.lse_out[orow(r)] = rowlse[r] * kLn2;
                } else {
                    float4 *dst = reinterpret_cast<float4 *>(p.o_part + (pslot * R + r) * D + d0);
                    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
                    if (d0 == 0) p.lse_part[pslot * R + r] = rowlse[r];
                }
            }
        };

        if constexpr (CC == 0) {
            // This warp's row group: rows rbase .. rbase + 8 * NTW - 1 (all rows
            // unless the unit has 32, when warps 0, 1 take rows 0-15 and warps 2,
            // 3 rows 16-31)
            const int rg = warp / C::GW;
            const int rbase = 16 * rg;
            // visible token range [lo, hi) of the two query rows this lane holds
            // per n-tile (rows rbase + 8*nt + 2*t4 + {0, 1}; row = query token * g
            // + head)
            int vis_lo[C::NTW][2], vis_hi[C::NTW][2];
#pragma unroll
            for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int row = rbase + nt * 8 + 2 * t4 + e;
                    const int hi = ctx - p.q_len + 1 + row / g;
                    vis_hi[nt][e] = row < R ? hi : 0;
                    vis_lo[nt][e] = (row < R && p.window > 0) ? max(0, hi - p.window) : 0;
                }

            // query fragments (B operand, Q^T[d][row]) from the slot: into
            // registers now, or (head_dim 256) by ldmatrix at every k-step
            const uint32_t qbase = sQ + qs * C::QSLOT;
            uint32_t qf[C::QSMEM ? 1 : C::KSTEPS][C::NTW][2];
            if constexpr (!C::QSMEM) {
                const uint32_t qb = qbase;
#pragma unroll
                for (int nt = 0; nt < C::NTW; ++nt) {
                    const int head = rbase + nt * 8 + gid;   // query row held as B column
                    const bool live = head < R;
                    const uint32_t qr = qb + (live ? head : 0) * C::QROW;
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k) {
                        uint32_t b0, b1;
                        if (!FP8) {   // k index 2t, 2t+1 | 2t+8, 2t+9  <->  same d
                            b0 = lds32(qr + (16 * k + 2 * t4) * 2);
                            b1 = lds32(qr + (16 * k + 8 + 2 * t4) * 2);
                        } else {      // k index permuted to d = 16k + 4t + {0,1 | 2,3}:
                            // 4 consecutive bf16, converted to f16 below
                            const long long v = lds64(qr + (16 * k + 4 * t4) * 2);
                            b0 = (uint32_t)v;
                            b1 = (uint32_t)((unsigned long long)v >> 32);
                        }
                        qf[k][nt][0] = live ? b0 : 0u;
                        qf[k][nt][1] = live ? b1 : 0u;
                    }
                }
                if constexpr (FP8) {
                    // The FP8 product runs in f16 (every E4M3 value is an f16
                    // value), whose range is narrower than bf16's.  The unit's
                    // query rows are scaled by a power of two 2^sh that puts their
                    // largest magnitude in [2^14, 2^15), so no value overflows and
                    // small ones keep their bits, and the score scale takes 2^-sh
                    // back (both exact).  The warps of a row group read the same
                    // rows, so they pick the same sh.
                    float qmax = 0.f;
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k)
#pragma unroll
                        for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float2 f = unpack_bf16x2(qf[k][nt][e]);
                                qmax = fmaxf(qmax, fmaxf(fabsf(f.x), fabsf(f.y)));
                            }
#pragma unroll
                    for (int off = 16; off; off >>= 1)
                        qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, off));
                    const int ex = qmax > 0.f ? (int)((__float_as_uint(qmax) >> 23) & 0xffu) - 127 : 14;
                    const int sh = min(100, max(-100, 14 - ex));
                    const float up = __uint_as_float((uint32_t)(127 + sh) << 23);
                    sl2 *= __uint_as_float((uint32_t)(127 - sh) << 23);
#pragma unroll
                    for (int k = 0; k < C::KSTEPS; ++k)
#pragma unroll
                        for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float2 f = unpack_bf16x2(qf[k][nt][e]);
                                qf[k][nt][e] = pack_f16x2(f.x * up, f.y * up);
                            }
                }
            }
            if (!C::QSMEM) {
                __syncwarp();
                if (lane == 0) mbar_arrive(seg_empty + 8 * qs);   // the slot may be refilled
            }
            ++sit;

            // This warp's online-softmax state over its own tokens of every
            // stage (16, or 32 with two row groups): running max and
            // (lane-partial) sum per query row, and O^T[d][row] for all D dims.
            // The states of a row group's warps are merged once, at the end of
            // the segment.
            float m_run[C::NTW][2], l_run[C::NTW][2];
            float o[C::DT][C::NTW][4];
#pragma unroll
            for (int nt = 0; nt < C::NTW; ++nt) {
                m_run[nt][0] = m_run[nt][1] = -INFINITY;
                l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
                for (int mt = 0; mt < C::DT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[mt][nt][e] = 0.f;
            }

            bool abort = false;
            for (int jj = j0; jj < j1; jj += C::BPS) {
                const int nb = min(C::BPS, j1 - jj);
                // tokens of the stage that were loaded (the stage may end with the
                // segment or with the context)
                const int n_valid = min(ctx - jj * BS, nb * BS);
                const uint32_t slot = it % NSTAGES;
                const bool ok = mbar_wait_bounded(bar_full + 8 * slot, (it / NSTAGES) & 1, p.wait_ns);
                ++it;
                if (!ok) {
                    raise_flag(p.flags, kFlagTimeout);
                    abort = true;
                    break;
                }
                const uint32_t sK = sbase + slot * C::STAGE, sV = sK + C::STAGE_KV;

                // this warp's 16-token sub-tiles: its own 16 (or 32) tokens of the stage
                for (int sub = 0; sub < C::SUBS; ++sub) {
                    // first stage token of this warp's 16-token sub-tile
                    const int tb = C::RG == 1 ? 16 * warp : 32 * (warp & 1) + 16 * sub;
                    if (tb < n_valid) {
                        // ---- S^T = K . Q^T for this warp's 16 tokens (two MMA chains)
                        float sacc[C::NTW][4], sac2[C::NTW][4];
#pragma unroll
                        for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                            for (int e = 0; e < 4; ++e) sacc[nt][e] = sac2[nt][e] = 0.f;
                        if (!FP8) {
                            const int mi = lane >> 3;
                            const int tok = tb + (mi & 1) * 8 + (lane & 7);
                            const int row = tok % BS;
                            const uint32_t rowaddr = sK + (tok / BS) * C::TILE + row * 128;
                            uint32_t qb4[C::NTW][4];   // shared-memory query fragments of k, k + 1
#pragma unroll
                            for (int k = 0; k < C::KSTEPS; ++k) {
                                const int chunk = 2 * k + (mi >> 1);
                                const uint32_t addr = rowaddr + (chunk >> 3) * (BS * 128) +
                                                      (((chunk & 7) ^ (row & 7)) << 4);
                                uint32_t a0, a1, a2, a3;
                                ldsm_x4(addr, a0, a1, a2, a3);
                                if constexpr (C::QSMEM) {
                                    if ((k & 1) == 0) {
                                        // matrices: rows nt*8 .. +7 at d = 16k, 16k+8, 16k+16, 16k+24
#pragma unroll
                                        for (int nt = 0; nt < C::NTW; ++nt)
                                            ldsm_x4(qbase + (rbase + nt * 8 + (lane & 7)) * C::QROW +
                                                        (16 * (k + (lane >> 4)) + 8 * ((lane >> 3) & 1)) * 2,
                                                    qb4[nt][0], qb4[nt][1], qb4[nt][2], qb4[nt][3]);
                                    }
                                }
#pragma unroll
                                for (int nt = 0; nt < C::NTW; ++nt) {
                                    uint32_t b0, b1;
                                    if constexpr (C::QSMEM) {
                                        b0 = qb4[nt][(k & 1) * 2];
                                        b1 = qb4[nt][(k & 1) * 2 + 1];
                                    } else {
                                        b0 = qf[k][nt][0];
                                        b1 = qf[k][nt][1];
                                    }
                                    if (k & 1) mma_bf16(sac2[nt], a0, a1, a2, a3, b0, b1);
                                    else       mma_bf16(sacc[nt], a0, a1, a2, a3, b0, b1);
                                }
                            }
                        } else {
                            const int tok0 = tb + gid, tok1 = tok0 + 8;
                            const int r0 = tok0 % BS, r1 = tok1 % BS;
                            const uint32_t base0 = sK + (tok0 / BS) * C::TILE + r0 * 128 + 4 * t4;
                            const uint32_t base1 = sK + (tok1 / BS) * C::TILE + r1 * 128 + 4 * t4;
#pragma unroll
                            for (int k = 0; k < C::KSTEPS; ++k) {
                                const uint32_t w0 = lds32(base0 + ((k ^ (r0 & 7)) << 4));
                                const uint32_t w1 = lds32(base1 + ((k ^ (r1 & 7)) << 4));
                                const uint32_t a0 = e4m3x2_to_f16x2(w0 & 0xffffu);
                                const uint32_t a2 = e4m3x2_to_f16x2(w0 >> 16);
                                const uint32_t a1 = e4m3x2_to_f16x2(w1 & 0xffffu);
                                const uint32_t a3 = e4m3x2_to_f16x2(w1 >> 16);
#pragma unroll
                                for (int nt = 0; nt < C::NTW; ++nt) {
                                    if (k & 1) mma_f16(sac2[nt], a0, a1, a2, a3, qf[k][nt][0], qf[k][nt][1]);
                                    else       mma_f16(sacc[nt], a0, a1, a2, a3, qf[k][nt][0], qf[k][nt][1]);
                                }
                            }
                        }

                        // ---- mask, this warp's max per row, weights p ----------------
                        float mx[C::NTW][2], alpha[C::NTW][2];
#pragma unroll
                        for (int nt = 0; nt < C::NTW; ++nt) {
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                // stage token (only the first n_valid were loaded) and
                                // its absolute position; the row's visible range
                                // excludes padding rows and positions past ctx
                                const int tok = tb + gid + (e >> 1) * 8;
                                const int pos = jj * BS + tok;
                                const float v = sacc[nt][e] + sac2[nt][e];
                                sacc[nt][e] = (tok < n_valid && pos >= vis_lo[nt][e & 1] &&
                                               pos < vis_hi[nt][e & 1])
                                                  ? v * sl2 : -INFINITY;
                            }
                            mx[nt][0] = fmaxf(sacc[nt][0], sacc[nt][2]);
                            mx[nt][1] = fmaxf(sacc[nt][1], sacc[nt][3]);
#pragma unroll
                            for (int off = 4; off < 32; off <<= 1) {
                                mx[nt][0] = fmaxf(mx[nt][0], __shfl_xor_sync(0xffffffffu, mx[nt][0], off));
                                mx[nt][1] = fmaxf(mx[nt][1], __shfl_xor_sync(0xffffffffu, mx[nt][1], off));
                            }
                        }
                        // Lazy rescaling: a row keeps its reference max m_run (the
                        // exponent offset of every weight it has summed) until a
                        // score exceeds it by more than 2^8, so weights stay below
                        // 256 and the accumulator is rescaled only in the stages
                        // where some row of the warp moves.
                        bool moved = false;
#pragma unroll
                        for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                            for (int e = 0; e < 2; ++e)
                                moved |= mx[nt][e] > m_run[nt][e] + kLazyRescale;
                        const bool any_moved = __any_sync(0xffffffffu, moved);
#pragma unroll
                        for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                alpha[nt][e] = 1.f;
                                if (any_moved && mx[nt][e] > m_run[nt][e] + kLazyRescale) {
                                    alpha[nt][e] = ex2(m_run[nt][e] - mx[nt][e]);
                                    m_run[nt][e] = mx[nt][e];
                                }
                                mx[nt][e] = m_run[nt][e] == -INFINITY ? 0.f : m_run[nt][e];
                            }
                        // rows past the end of the context may hold anything (NaN,
                        // Inf): zero this warp's invalid V rows so that 0 * V stays 0
                        if (n_valid < tb + 16) {
                            const int first = max(tb, n_valid), last = tb + 16;
                            const int lines = (last - first) * C::LINES;
                            for (int i = lane >> 3; i < lines; i += 4) {
                                const int tok = first + i / C::LINES, ln = i % C::LINES;
                                const uint32_t a = sV + (tok / BS) * C::TILE + ln * (BS * 128) +
                                                   (tok % BS) * 128 + (lane & 7) * 16;
                                sts128(a, 0u, 0u, 0u, 0u);
                            }
                            // order these generic-proxy writes before the next TMA
                            // into the slot
                            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                            __syncwarp();
                        }

                        // ---- P^T fragments (B operand, k = token, n = row) ------------
                        // The score accumulator holds S^T[token][row] in the fragment
                        // layout (lane 4r + c: tokens r and r + 8, rows 2c, 2c + 1); a
                        // warp transpose of each 8x8 half gives P^T[row][token] in
                        // the B-operand layout of the PV product.
                        uint32_t pb[C::NTW][2], pl[C::NTW][2];
#pragma unroll
                        for (int nt = 0; nt < C::NTW; ++nt) {
                            float pr[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) pr[e] = ex2(sacc[nt][e] - mx[nt][e & 1]);
                            if (!FP8) {
                                // p = hi + lo, both bf16; the normaliser sums the fp32 p
                                const uint32_t h0 = pack_bf16x2(pr[0], pr[1]);
                                const uint32_t h1 = pack_bf16x2(pr[2], pr[3]);
                                const float2 q0 = unpack_bf16x2(h0), q1 = unpack_bf16x2(h1);
                                const uint32_t l0 = pack_bf16x2(pr[0] - q0.x, pr[1] - q0.y);
                                const uint32_t l1 = pack_bf16x2(pr[2] - q1.x, pr[3] - q1.y);
                                l_run[nt][0] = l_run[nt][0] * alpha[nt][0] + pr[0] + pr[2];
                                l_run[nt][1] = l_run[nt][1] * alpha[nt][1] + pr[1] + pr[3];
                                pb[nt][0] = movmatrix_trans(h0);
                                pb[nt][1] = movmatrix_trans(h1);
                                pl[nt][0] = movmatrix_trans(l0);
                                pl[nt][1] = movmatrix_trans(l1);
                            } else {
                                // f16 weights; the normaliser sums exactly the rounded values
                                const uint32_t h0 = pack_f16x2(pr[0], pr[1]);
                                const uint32_t h1 = pack_f16x2(pr[2], pr[3]);
                                const float2 q0 = unpack_f16x2(h0), q1 = unpack_f16x2(h1);
                                l_run[nt][0] = l_run[nt][0] * alpha[nt][0] + q0.x + q1.x;
                                l_run[nt][1] = l_run[nt][1] * alpha[nt][1] + q0.y + q1.y;
                                pb[nt][0] = movmatrix_trans(h0);
                                pb[nt][1] = movmatrix_trans(h1);
                            }
                        }

                        // ---- O^T += V^T . P^T over all D for this warp's tokens ------
                        if (any_moved) {
#pragma unroll
                            for (int mt = 0; mt < C::DT; ++mt)
#pragma unroll
                                for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                                    for (int e = 0; e < 4; ++e) o[mt][nt][e] *= alpha[nt][e & 1];
                        }
                        if (!FP8) {
                            const int mi = lane >> 3;
                            const int tok = tb + (mi >> 1) * 8 + (lane & 7);
                            const int row = tok % BS;
                            const uint32_t rowaddr = sV + (tok / BS) * C::TILE + row * 128;
#pragma unroll
                            for (int mt = 0; mt < C::DT; ++mt) {
                                const int chunk = 2 * mt + (mi & 1);
                                const uint32_t addr = rowaddr + (chunk >> 3) * (BS * 128) +
                                                      (((chunk & 7) ^ (row & 7)) << 4);
                                uint32_t a0, a1, a2, a3;
                                ldsm_x4_t(addr, a0, a1, a2, a3);
#pragma unroll
                                for (int nt = 0; nt < C::NTW; ++nt) {
                                    mma_bf16(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
                                    mma_bf16(o[mt][nt], a0, a1, a2, a3, pl[nt][0], pl[nt][1]);
                                }
                            }
                        } else {
                            // tokens 2c, 2c+1, 2c+8, 2c+9 of this warp; 16 bytes at
                            // d = 16*gid .. 16*gid + 15 (m-tile mt: bytes 2mt, 2mt+1)
                            uint32_t wv[4][4];
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const int tok = tb + 2 * t4 + (q & 1) + (q >> 1) * 8;
                                const int row = tok % BS;
                                lds128(sV + (tok / BS) * C::TILE + row * 128 + ((gid ^ (row & 7)) << 4),
                                       wv[q][0], wv[q][1], wv[q][2], wv[q][3]);
                            }
#pragma unroll
                            for (int mt = 0; mt < C::DT; ++mt) {
                                const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
                                const uint32_t x = prmt(wv[0][mt >> 1], wv[1][mt >> 1], sel);
                                const uint32_t y = prmt(wv[2][mt >> 1], wv[3][mt >> 1], sel);
                                const uint32_t a0 = e4m3x2_to_f16x2(x & 0xffffu);
                                const uint32_t a1 = e4m3x2_to_f16x2(x >> 16);
                                const uint32_t a2 = e4m3x2_to_f16x2(y & 0xffffu);
                                const uint32_t a3 = e4m3x2_to_f16x2(y >> 16);
#pragma unroll
                                for (int nt = 0; nt < C::NTW; ++nt)
                                    mma_f16(o[mt][nt], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_empty + 8 * slot);
            }
            if (C::QSMEM) {
                __syncwarp();
                if (lane == 0) mbar_arrive(seg_empty + 8 * qs);   // query rows read
            }

            // ---- finish the segment: merge the warps' states -------------------
            // In a fixed order, so that results do not depend on timing.  With one
            // row group, warps 1 and 3 store their O rows (buffers A and B), warps
            // 0 and 2 add theirs to them with both weights, and the output is
            // (A + B) / L.  With two row groups (32 rows), each group's odd warp
            // stores, its even warp adds, and the output is that buffer / L.
            // output dim held by accumulator element (mt, e)
            auto dim_of = [&](int mt, int e) -> int {
                if (!FP8) return 16 * mt + gid + (e >> 1) * 8;
                return 16 * gid + 2 * mt + (e >> 1);
            };
            // A: warps 0, 1; B: warps 2, 3
            auto store_rows = [&](int nt) {
                float *buf = reinterpret_cast<float *>(
                    smem + C::OFF_O + (C::NOBUF == 2 ? (warp >> 1) : 0) * C::OBUF);
#pragma unroll
                for (int mt = 0; mt < C::DT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        buf[(2 * t4 + (e & 1)) * C::OROW + dim_of(mt, e)] = o[mt][nt][e];
            };
            if ((warp & 1) && rg == 0) store_rows(0);
            // row sums over this warp's lanes; row max and sum of every warp
            // through shared memory; all consumers agree on leaving after a timeout
#pragma unroll
            for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = l_run[nt][e];
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                    if (gid == 0) {
                        red[warp * C::NP + rbase + nt * 8 + 2 * t4 + e] = m_run[nt][e];
                        lsum[warp * C::NP + rbase + nt * 8 + 2 * t4 + e] = v;
                    }
                }
            if (named_bar_sync_or(kBarConsumers, kConsumers, abort)) return;
            // weights of this warp's and its partner's (warp + 1) O in the merged
            // row; the row's max and sum run over the warps of its row group
            const int w0 = rg * C::GW;
            float wsc[C::NTW][2], psc[C::NTW][2];
#pragma unroll
            for (int nt = 0; nt < C::NTW; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int r = rbase + nt * 8 + 2 * t4 + e;
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < C::GW; ++w) M = fmaxf(M, red[(w0 + w) * C::NP + r]);
                    const float Mu = M == -INFINITY ? 0.f : M;
                    wsc[nt][e] = ex2(m_run[nt][e] - Mu);
                    psc[nt][e] = ex2(red[((warp + 1) & 3) * C::NP + r] - Mu);
                    if (warp == w0 && gid == 0) {
                        float L = 0.f;
#pragma unroll
                        for (int w = 0; w < C::GW; ++w)
                            L += lsum[(w0 + w) * C::NP + r] * ex2(red[(w0 + w) * C::NP + r] - Mu);
                        rowinv[r] = L > 0.f ? vsc / L : 0.f;
                        rowlse[r] = L > 0.f ? M + log2f(L) : -INFINITY;
                    }
                }

            // Rounds of 8 rows: with two buffers both halves of the warps merge
            // rows 8*nt .. 8*nt + 7 together (A: warps 0, 1; B: warps 2, 3); with
            // two row groups one buffer serves the group of the round.
#pragma unroll
            for (int rd = 0; rd < C::RG * C::NTW; ++rd) {
                const int grp = rd / C::NTW, nt = rd % C::NTW;
                if (rd > 0) {
                    named_bar_sync(kBarConsumers, kConsumers);   // buffers read
                    if ((warp & 1) && rg == grp) store_rows(nt);
                    named_bar_sync(kBarConsumers, kConsumers);
                }
                // even warps: buffer = own O * weight + partner's O * its weight
                if (!(warp & 1) && rg == grp) {
                    float *buf = reinterpret_cast<float *>(
                        smem + C::OFF_O + (C::NOBUF == 2 ? (warp >> 1) : 0) * C::OBUF);
                    float part[C::DT][4];
#pragma unroll
                    for (int mt = 0; mt < C::DT; ++mt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            part[mt][e] = buf[(2 * t4 + (e & 1)) * C::OROW + dim_of(mt, e)];
#pragma unroll
                    for (int mt = 0; mt < C::DT; ++mt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            buf[(2 * t4 + (e & 1)) * C::OROW + dim_of(mt, e)] =
                                o[mt][nt][e] * wsc[nt][e & 1] + part[mt][e] * psc[nt][e & 1];
                }
                named_bar_sync(kBarConsumers, kConsumers);
                finalize_rows(grp * 16 + nt * 8);
            }
        } else {
            // ---- CUDA-core variant: FMA dot products, warp-shuffle sums --------
            // Lane l owns dims 4l .. 4l+3 of every query row (head_dim 128).
            // For a group of TG tokens each lane forms the partial dot products
            // of its 4 dims for all TG x CC (token, row) pairs; a butterfly of
            // shuffles leaves lane l the full score of pair l (token l / CC,
            // row l % CC).  P goes through this warp's shared-memory area to
            // every lane, which accumulates O for its 4 dims of every row.
            constexpr int RP = CC, TG = 32 / RP, NGR = 16 / TG;
            const int my_r = lane % RP;            // the row of the scores this lane holds
            int vlo, vhi;
            {
                const int hi = ctx - p.q_len + 1 + my_r / g;
                vhi = my_r < R ? hi : 0;
                vlo = (my_r < R && p.window > 0) ? max(0, hi - p.window) : 0;
            }
            // dims 4l .. 4l+3 of bf16 row `tok` of a K or V stage, as fp32
            auto load4 = [&](uint32_t tile0, int tok, float (&v)[4]) {
                const int row = tok % BS;
                const uint32_t a = tile0 + (tok / BS) * C::TILE + (lane >> 4) * (BS * 128) +
                                   row * 128 + ((((lane & 15) >> 1) ^ (row & 7)) << 4) +
                                   8 * (lane & 1);
                const long long w = lds64(a);
                const uint32_t x = (uint32_t)w, y = (uint32_t)(w >> 32);
                v[0] = __uint_as_float(x << 16);
                v[1] = __uint_as_float(x & 0xFFFF0000u);
                v[2] = __uint_as_float(y << 16);
                v[3] = __uint_as_float(y & 0xFFFF0000u);
            };
            float qv[RP][4];
            {
                const uint32_t qb = sQ + qs * C::QSLOT;
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const long long w = lds64(qb + (min(r, R - 1) * D + 4 * lane) * 2);
                    const uint32_t x = (uint32_t)w, y = (uint32_t)(w >> 32);
                    const bool live = r < R;
                    qv[r][0] = live ? __uint_as_float(x << 16) : 0.f;
                    qv[r][1] = live ? __uint_as_float(x & 0xFFFF0000u) : 0.f;
                    qv[r][2] = live ? __uint_as_float(y << 16) : 0.f;
                    qv[r][3] = live ? __uint_as_float(y & 0xFFFF0000u) : 0.f;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(seg_empty + 8 * qs);   // the slot may be refilled
            ++sit;

            float o4[RP][4];
#pragma unroll
            for (int r = 0; r < RP; ++r)
#pragma unroll
                for (int j = 0; j < 4; ++j) o4[r][j] = 0.f;
            float m_my = -INFINITY, l_my = 0.f;   // this lane's row: running max, its share of the sum
            float *pw = reinterpret_cast<float *>(smem + C::OFF_PW) + warp * C::PWF;
            bool abort = false;
            for (int jj = j0; jj < j1; jj += C::BPS) {
                const int nb = min(C::BPS, j1 - jj);
                const int n_valid = min(ctx - jj * BS, nb * BS);
                const uint32_t slot = it % NSTAGES;
                const bool ok = mbar_wait_bounded(bar_full + 8 * slot, (it / NSTAGES) & 1, p.wait_ns);
                ++it;
                if (!ok) {
                    raise_flag(p.flags, kFlagTimeout);
                    abort = true;
                    break;
                }
                const uint32_t sK = sbase + slot * C::STAGE, sV = sK + C::STAGE_KV;
                const int nv = n_valid - 16 * warp;   // loaded tokens of this warp (uniform)
                if (nv > 0) {
                    float sc[NGR];
#pragma unroll
                    for (int gi = 0; gi < NGR; ++gi) {
                        float acc[32];
#pragma unroll
                        for (int tt = 0; tt < TG; ++tt) {
                            const int tk = gi * TG + tt;
                            float k4[4] = {0.f, 0.f, 0.f, 0.f};
                            if (tk < nv) load4(sK, 16 * warp + tk, k4);
#pragma unroll
                            for (int r = 0; r < RP; ++r)
                                acc[tt * RP + r] = qv[r][0] * k4[0] + qv[r][1] * k4[1] +
                                                   qv[r][2] * k4[2] + qv[r][3] * k4[3];
                        }
                        // reduce-scatter over the 32 lanes: lane l keeps entry l
#pragma unroll
                        for (int off = 16, len = 32; off >= 1; off >>= 1, len >>= 1) {
                            const bool up = (lane & off) != 0;
#pragma unroll
                            for (int i = 0; i < len / 2; ++i) {
                                const float send = up ? acc[i] : acc[i + len / 2];
                                const float keep = up ? acc[i + len / 2] : acc[i];
                                acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                            }
                        }
                        const int tk = gi * TG + lane / RP;
                        const int pos = jj * BS + 16 * warp + tk;
                        sc[gi] = (tk < nv && pos >= vlo && pos < vhi) ? acc[0] * sl2 : -INFINITY;
                    }
                    // this stage's max of the lane's row (lanes with the same row)
                    float mx = sc[0];
#pragma unroll
                    for (int gi = 1; gi < NGR; ++gi) mx = fmaxf(mx, sc[gi]);
#pragma unroll
                    for (int off = RP; off < 32; off <<= 1)
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    const float m_new = fmaxf(m_my, mx);
                    const float m_use = m_new == -INFINITY ? 0.f : m_new;
                    const float al = ex2(m_my - m_use);
                    m_my = m_new;
                    float ps = 0.f;
#pragma unroll
                    for (int gi = 0; gi < NGR; ++gi) {
                        const float pv = ex2(sc[gi] - m_use);
                        ps += pv;
                        pw[(gi * TG + lane / RP) * RP + my_r] = pv;
                    }
                    l_my = l_my * al + ps;
                    if (lane < RP) pw[16 * RP + lane] = al;
                    __syncwarp();
                    // rescale O and add this warp's tokens
#pragma unroll
                    for (int r = 0; r < RP; ++r) {
                        const float a = pw[16 * RP + r];
#pragma unroll
                        for (int j = 0; j < 4; ++j) o4[r][j] *= a;
                    }
                    for (int tk = 0; tk < min(nv, 16); ++tk) {
                        float v4[4];
                        load4(sV, 16 * warp + tk, v4);
#pragma unroll
                        for (int r4 = 0; r4 < RP / 4; ++r4) {
                            const float4 pr = reinterpret_cast<const float4 *>(pw + tk * RP)[r4];
                            const float pp[4] = {pr.x, pr.y, pr.z, pr.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i)
#pragma unroll
                                for (int j = 0; j < 4; ++j) o4[4 * r4 + i][j] += pp[i] * v4[j];
                        }
                    }
                    __syncwarp();   // pw is rewritten by the next stage
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_empty + 8 * slot);
            }

            // ---- merge the 4 warps' states (same fixed order as above) --------
            float *buf = reinterpret_cast<float *>(smem + C::OFF_O + (warp >> 1) * C::OBUF);
            if (warp & 1) {
#pragma unroll
                for (int r = 0; r < RP; ++r)
                    *reinterpret_cast<float4 *>(buf + r * C::OROW + 4 * lane) =
                        make_float4(o4[r][0], o4[r][1], o4[r][2], o4[r][3]);
            }
            float lr = l_my;
#pragma unroll
            for (int off = RP; off < 32; off <<= 1) lr += __shfl_xor_sync(0xffffffffu, lr, off);
            if (lane < C::NP) {       // lane r < RP holds row r
                red[warp * C::NP + lane] = lane < RP ? m_my : -INFINITY;
                lsum[warp * C::NP + lane] = lane < RP ? lr : 0.f;
            }
            if (named_bar_sync_or(kBarConsumers, kConsumers, abort)) return;
            float wsc[RP], psc[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red[w * C::NP + r]);
                const float Mu = M == -INFINITY ? 0.f : M;
                wsc[r] = ex2(red[warp * C::NP + r] - Mu);
                psc[r] = ex2(red[((warp + 1) & 3) * C::NP + r] - Mu);
            }
            if (warp == 0 && lane < C::NP) {
                const int r = lane;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red[w * C::NP + r]);
                const float Mu = M == -INFINITY ? 0.f : M;
                float L = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w)
                    L += lsum[w * C::NP + r] * ex2(red[w * C::NP + r] - Mu);
                rowinv[r] = L > 0.f ? vsc / L : 0.f;
                rowlse[r] = L > 0.f ? M + log2f(L) : -INFINITY;
            }
            if (!(warp & 1)) {
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    float4 *b4 = reinterpret_cast<float4 *>(buf + r * C::OROW + 4 * lane);
                    const float4 q4 = *b4;
                    *b4 = make_float4(o4[r][0] * wsc[r] + q4.x * psc[r],
                                      o4[r][1] * wsc[r] + q4.y * psc[r],
                                      o4[r][2] * wsc[r] + q4.z * psc[r],
                                      o4[r][3] * wsc[r] + q4.w * psc[r]);
                }
            }
            named_bar_sync(kBarConsumers, kConsumers);
            finalize_rows(0);
        }
        if (!whole) {
            // every consumer's partial stores precede the barrier; the arrival
            // count is an acquire-release atomic, so the last CTA to arrive
            // sees all pieces (the barriers carry the ordering to the other
            // threads of both CTAs)
            named_bar_sync(kBarConsumers, kConsumers);
            // unit tile range [ua, ub) in work space and the CTAs that share it
            const long long ua = useg - (j0 - jlo);
            const long long ub = ua + (nunit - jlo);
            const long long c_first = cta_of(ua, U, G), c_last = cta_of(ub - 1, U, G);
            if (tid == 0) {
                const int prev = atom_add_acq_rel_gpu(p.counters + (long long)s * Hkv + h, 1);
                misc->is_last = (prev == (int)(c_last - c_first));
            }
            named_bar_sync(kBarConsumers, kConsumers);
            if (misc->is_last) {
                merge_unit<D>(p, ua, U, G, c_first, c_last, s, h);
                if (tid == 0) p.counters[(long long)s * Hkv + h] = 0;
            }
        }
    }
}

}  // namespace pgd
