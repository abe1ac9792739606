// pgd_aux.cu -- the KV append scatter and the standalone log-sum-exp merge.
#include "pgd_launch.h"

namespace pgd {

// Copy the K and V rows (head_dim elements of the cache type) of each (new
// token, KV head) into physical block slot / bs, row slot % bs ("batching and
// attention" 3.4: KV lives in fixed-size blocks).  A (token, head) pair is
// 2 * row_vec 16-byte chunks, K's then V's; one lane moves one chunk, so a
// warp serves one pair of 512-byte rows (bf16, head_dim 128), or two pairs of
// 256-byte rows (FP8), or one pair in two passes (head_dim 256).  The copy is
// bit-exact.
__global__ void __launch_bounds__(256)
kv_append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                 const int64_t *__restrict__ slots, int32_t num_tokens, uint4 *k_cache,
                 uint4 *v_cache, int32_t hkv, int32_t row_vec, int32_t bs, int64_t pool_slots,
                 uint32_t *flags) {
    const int cp = 2 * row_vec;                  // chunks of one (token, head) pair
    const int lp = cp < 32 ? cp : 32;            // lanes per pair
    const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long pair = gw * (32 / lp) + lane / lp;
    const int sub = lane % lp;
    if (pair >= static_cast<long long>(num_tokens) * hkv) return;
    const int t = static_cast<int>(pair / hkv), h = static_cast<int>(pair % hkv);
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) return;                       // padding token
    if (slot >= pool_slots) {
        if (sub == 0 && h == 0) raise_flag(flags, kFlagSlot);
        return;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    const int64_t src = (static_cast<int64_t>(t) * hkv + h) * row_vec;
    const int64_t dst = ((blk * hkv + h) * bs + off) * row_vec;
    for (int c = sub; c < cp; c += lp) {
        const bool isk = c < row_vec;
        const int ch = isk ? c : c - row_vec;
        (isk ? k_cache : v_cache)[dst + ch] = __ldg((isk ? k_new : v_new) + src + ch);
    }
}

cudaError_t launch_kv_append(const void *k_new, const void *v_new, const int64_t *slots,
                             int32_t num_tokens, void *k_cache, void *v_cache, int32_t hkv,
                             int32_t row_bytes, int32_t block_size, int64_t pool_slots,
                             uint32_t *flags, cudaStream_t stream) {
    const int row_vec = row_bytes / 16;
    const int lp = 2 * row_vec < 32 ? 2 * row_vec : 32;
    const long long pairs = static_cast<long long>(num_tokens) * hkv;
    const long long warps = (pairs * lp + 31) / 32;
    const long long blocks = (warps * 32 + 255) / 256;
    kv_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slots, num_tokens,
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), hkv, row_vec, block_size,
        pool_slots, flags);
    return cudaGetLastError();
}

// Quantising append: bf16 K/V rows of new tokens into an FP8 E4M3 cache
// ("attention kernels", "what to check": FP8 KV).  Each element is divided by
// its KV head's fp32 scale (IEEE division) and rounded to E4M3.  One warp per
// (token, KV head); each lane turns 8 bf16 (16 bytes) into 8 bytes.
__global__ void __launch_bounds__(256)
kv_append_quant_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                       const int64_t *__restrict__ slots, int32_t num_tokens, uint2 *k_cache,
                       uint2 *v_cache, const float *__restrict__ k_scale,
                       const float *__restrict__ v_scale, int32_t hkv, int32_t row_vec,
                       int32_t bs, int64_t pool_slots, uint32_t *flags) {
    const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= static_cast<long long>(num_tokens) * hkv) return;
    const int t = static_cast<int>(w / hkv), h = static_cast<int>(w % hkv);
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) return;
    if (slot >= pool_slots) {
        if (lane == 0 && h == 0) raise_flag(flags, kFlagSlot);
        return;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    const int64_t src = (static_cast<int64_t>(t) * hkv + h) * row_vec;      // in uint4
    const int64_t dst = ((blk * hkv + h) * bs + off) * row_vec;             // in uint2
    const float ks = __ldg(k_scale + h), vs = __ldg(v_scale + h);
    for (int c = lane; c < 2 * row_vec; c += 32) {
        const bool isk = c < row_vec;
        const int ch = isk ? c : c - row_vec;
        const uint4 x = __ldg((isk ? k_new : v_new) + src + ch);
        const float s = isk ? ks : vs;
        const uint32_t in[4] = {x.x, x.y, x.z, x.w};
        uint32_t b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = unpack_bf16x2(in[i]);
            b[i] = f32x2_to_e4m3x2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
        }
        (isk ? k_cache : v_cache)[dst + ch] = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
    }
}

cudaError_t launch_kv_append_quant(const void *k_new, const void *v_new, const int64_t *slots,
                                   int32_t num_tokens, void *k_cache, void *v_cache,
                                   const float *k_scale, const float *v_scale, int32_t hkv,
                                   int32_t head_dim, int32_t block_size, int64_t pool_slots,
                                   uint32_t *flags, cudaStream_t stream) {
    const long long warps = static_cast<long long>(num_tokens) * hkv;
    const long long blocks = (warps * 32 + 255) / 256;
    kv_append_quant_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slots, num_tokens,
        static_cast<uint2 *>(k_cache), static_cast<uint2 *>(v_cache), k_scale, v_scale, hkv,
        head_dim / 8, block_size, pool_slots, flags);
    return cudaGetLastError();
}

// Merge of split results by log-sum-exp ("attention kernels", section
// "prefill and decode attention"): one warp per row, each lane holding one
// (head_dim 128) or two (256) float4 columns, the pieces read in order with
// several in flight.
//   M = max_p lse_p;  w_p = exp(lse_p - M);  out = sum w_p o_p / sum w_p.
constexpr int kMergeRowsPerCta = 4;

__global__ void __launch_bounds__(32 * kMergeRowsPerCta)
merge_partials_kernel(const float *__restrict__ o_part, const float *__restrict__ lse_part,
                      int32_t parts, int32_t rows, int32_t head_dim, uint16_t *out,
                      float *lse_out) {
    // programmatic dependent launch: the split results come from the
    // previous launch on the stream
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int r = blockIdx.x * kMergeRowsPerCta + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= rows) return;
    constexpr float kLog2e = 1.4426950408889634f;
    float M = -INFINITY;
    for (int p = lane; p < parts; p += 32) M = fmaxf(M, __ldg(lse_part + (long long)p * rows + r));
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float Mu = M == -INFINITY ? 0.f : M;
    const int V4 = head_dim / 4;
    float W = 0.f;
    float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
#pragma unroll 4
    for (int p = 0; p < parts; ++p) {
        const float w = ex2((__ldg(lse_part + (long long)p * rows + r) - Mu) * kLog2e);
        W += w;
        const float4 *src =
            reinterpret_cast<const float4 *>(o_part + ((long long)p * rows + r) * head_dim);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int c = lane + 32 * i;
            if (c < V4) {
                const float4 v = __ldg(src + c);
                acc[i].x += w * v.x; acc[i].y += w * v.y; acc[i].z += w * v.z; acc[i].w += w * v.w;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int c = lane + 32 * i;
        if (c < V4) {
            uint2 packed;
            packed.x = pack_bf16x2(W > 0.f ? acc[i].x / W : 0.f, W > 0.f ? acc[i].y / W : 0.f);
            packed.y = pack_bf16x2(W > 0.f ? acc[i].z / W : 0.f, W > 0.f ? acc[i].w / W : 0.f);
            *reinterpret_cast<uint2 *>(out + (long long)r * head_dim + 4 * c) = packed;
        }
    }
    if (lse_out && lane == 0) lse_out[r] = W > 0.f ? M + logf(W) : -INFINITY;
}

cudaError_t launch_merge_partials(const float *o_part, const float *lse_part, int32_t parts,
                                  int32_t rows, int32_t head_dim, uint16_t *out, float *lse_out,
                                  cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>((rows + kMergeRowsPerCta - 1) / kMergeRowsPerCta));
    cfg.blockDim = dim3(32 * kMergeRowsPerCta);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, merge_partials_kernel, o_part, lse_part, parts, rows, head_dim,
                              out, lse_out);
}

}  // namespace pgd
