// pgd_aux.cu -- the KV append scatter and the standalone log-sum-exp merge.
#include "pgd_launch.h"

namespace pgd {

// One warp per (new token, KV head): copy the K and V rows (head_dim
// elements of the cache type) into physical block slot / bs, row slot % bs
// ("batching and attention" 3.4: KV lives in fixed-size blocks).  Rows are
// moved as 16-byte vectors; the copy is bit-exact.
__global__ void __launch_bounds__(256)
kv_append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                 const int64_t *__restrict__ slots, int32_t num_tokens, uint4 *k_cache,
                 uint4 *v_cache, int32_t hkv, int32_t row_vec, int32_t bs, int64_t pool_slots,
                 uint32_t *flags) {
    const long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= static_cast<long long>(num_tokens) * hkv) return;
    const int t = static_cast<int>(w / hkv), h = static_cast<int>(w % hkv);
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) return;                       // padding token
    if (slot >= pool_slots) {
        if (lane == 0 && h == 0) raise_flag(flags, kFlagSlot);
        return;
    }
    const int64_t blk = slot / bs, off = slot % bs;
    const int64_t src = (static_cast<int64_t>(t) * hkv + h) * row_vec;
    const int64_t dst = ((blk * hkv + h) * bs + off) * row_vec;
    for (int c = lane; c < row_vec; c += 32) {
        k_cache[dst + c] = __ldg(k_new + src + c);
        v_cache[dst + c] = __ldg(v_new + src + c);
    }
}

cudaError_t launch_kv_append(const void *k_new, const void *v_new, const int64_t *slots,
                             int32_t num_tokens, void *k_cache, void *v_cache, int32_t hkv,
                             int32_t row_bytes, int32_t block_size, int64_t pool_slots,
                             uint32_t *flags, cudaStream_t stream) {
    const long long warps = static_cast<long long>(num_tokens) * hkv;
    const long long blocks = (warps * 32 + 255) / 256;
    kv_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slots, num_tokens,
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), hkv, row_bytes / 16,
        block_size, pool_slots, flags);
    return cudaGetLastError();
}

// Two fp32 values -> two E4M3 bytes (round to nearest even, saturating at
// +-448), lo in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
    uint32_t r;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %2, %1;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(r) : "f"(lo), "f"(hi));
    return r;
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
// "prefill and decode attention"): one CTA per row, threads over head_dim.
//   M = max_p lse_p;  w_p = exp(lse_p - M);  out = sum w_p o_p / sum w_p.
__global__ void __launch_bounds__(128)
merge_partials_kernel(const float *__restrict__ o_part, const float *__restrict__ lse_part,
                      int32_t parts, int32_t rows, int32_t head_dim, uint16_t *out,
                      float *lse_out) {
    // programmatic dependent launch: the split results come from the
    // previous launch on the stream
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int r = blockIdx.x;
    constexpr float kLog2e = 1.4426950408889634f;
    float M = -INFINITY;
    for (int p = 0; p < parts; ++p) M = fmaxf(M, __ldg(lse_part + (long long)p * rows + r));
    const float Mu = M == -INFINITY ? 0.f : M;
    for (int d = threadIdx.x; d < head_dim; d += blockDim.x) {
        float W = 0.f, acc = 0.f;
        for (int p = 0; p < parts; ++p) {
            const float l = __ldg(lse_part + (long long)p * rows + r);
            const float w = ex2((l - Mu) * kLog2e);
            W += w;
            acc += w * __ldg(o_part + ((long long)p * rows + r) * head_dim + d);
        }
        out[(long long)r * head_dim + d] =
            __bfloat16_as_ushort(__float2bfloat16_rn(W > 0.f ? acc / W : 0.f));
        if (lse_out && d == 0) lse_out[r] = W > 0.f ? M + logf(W) : -INFINITY;
    }
}

cudaError_t launch_merge_partials(const float *o_part, const float *lse_part, int32_t parts,
                                  int32_t rows, int32_t head_dim, uint16_t *out, float *lse_out,
                                  cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(rows));
    cfg.blockDim = dim3(128);
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
