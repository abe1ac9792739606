// pgd_aux.cu -- the KV append scatter and the standalone log-sum-exp merge.
#include "pgd_launch.h"

namespace pgd {

// Copy the K and V rows (head_dim elements of the cache type) of each (new
// token, KV head) into physical block slot / bs, row slot % bs ("batching and
// attention" 3.4: KV lives in fixed-size blocks).  One CTA per new token:
// its hkv pairs of rows are 2 * row_vec 16-byte chunks each (K's then V's),
// one thread per chunk and round.  The chunk count per pair (lg_cp) and the
// block size (lg_bs) are powers of two, so a chunk's head, row and block are
// shifts and masks.  The copy is bit-exact.
constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads)
kv_append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                 const int64_t *__restrict__ slots, uint4 *k_cache, uint4 *v_cache, int32_t hkv,
                 int32_t row_vec, int32_t lg_cp, int32_t lg_bs, int64_t pool_slots,
                 uint32_t *flags) {
    const int t = blockIdx.x;
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) return;                       // padding token
    if (slot >= pool_slots) {
        if (threadIdx.x == 0) raise_flag(flags, kFlagSlot);
        return;
    }
    const int64_t blk = slot >> lg_bs, off = slot & ((1 << lg_bs) - 1);
    const int n = hkv << lg_cp;                 // chunks of the token
    for (int i = threadIdx.x; i < n; i += kAppendThreads) {
        const int h = i >> lg_cp, c = i & ((1 << lg_cp) - 1);
        const bool isk = c < row_vec;
        const int ch = isk ? c : c - row_vec;
        const int64_t src = (static_cast<int64_t>(t) * hkv + h) * row_vec + ch;
        const int64_t dst = (((blk * hkv + h) << lg_bs) + off) * row_vec + ch;
        (isk ? k_cache : v_cache)[dst] = __ldg((isk ? k_new : v_new) + src);
    }
}

__host__ __forceinline__ int lg2_exact(int v) {   // log2 of a power of two, else -1
    if (v <= 0 || (v & (v - 1))) return -1;
    int l = 0;
    while ((1 << l) < v) ++l;
    return l;
}

cudaError_t launch_kv_append(const void *k_new, const void *v_new, const int64_t *slots,
                             int32_t num_tokens, void *k_cache, void *v_cache, int32_t hkv,
                             int32_t row_bytes, int32_t block_size, int64_t pool_slots,
                             uint32_t *flags, cudaStream_t stream) {
    const int row_vec = row_bytes / 16;
    const int lg_cp = lg2_exact(2 * row_vec), lg_bs = lg2_exact(block_size);
    if (lg_cp < 0 || lg_bs < 0 || (static_cast<long long>(hkv) << lg_cp) > (1LL << 30))
        return cudaErrorInvalidValue;
    if (num_tokens == 0) return cudaSuccess;
    kv_append_kernel<<<static_cast<unsigned>(num_tokens), kAppendThreads, 0, stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slots,
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), hkv, row_vec, lg_cp,
        lg_bs, pool_slots, flags);
    return cudaGetLastError();
}

// Two fp32 lanes in one 64-bit register for the paired FP32 instructions
// (fma.rn.f32x2 / mul.rn.f32x2: each lane rounds as the scalar instruction).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    return static_cast<uint64_t>(__float_as_uint(lo)) |
           (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float f2_lo(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float f2_hi(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// x / s rounded to nearest, the quotient IEEE division gives, for the 8
// elements of one chunk, from r = RN(1/s).  y0 = RN(x r) is within two ulps
// of x / s.  One correction y1 = RN(y0 + (x - y0 s) r), the remainder taken
// in one FMA, brings it within an ulp; from that faithful y1 the remainder is
// exact and a second correction gives the correctly rounded quotient
// (Markstein's theorem: P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Develop. 34(1), 1990).
// The steps need r normal, the remainders clear of underflow and the
// quotients clear of overflow: with |s| in [2^-40, 2^40] and every |x| in
// [2^-60, 2^60] all of that holds (quotients within [2^-100, 2^100]).  Any
// other chunk (zeros and subnormals, whose signs and codes IEEE division
// settles, non-finite values, extreme magnitudes or scales) divides with
// __fdiv_rn.  The steps run on pairs of elements.
__device__ __forceinline__ void div_by_scale8(float (&x)[8], float s, float r) {
    bool fast = fabsf(s) >= 0x1p-40f && fabsf(s) <= 0x1p40f;
#pragma unroll
    for (int i = 0; i < 8; ++i) fast = fast && fabsf(x[i]) >= 0x1p-60f && fabsf(x[i]) <= 0x1p60f;
    if (fast) {
        const uint64_t r2 = f2_pack(r, r), ns2 = f2_pack(-s, -s);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const uint64_t xv = f2_pack(x[i], x[i + 1]);
            const uint64_t y0 = f2_mul(xv, r2);
            const uint64_t y1 = f2_fma(f2_fma(y0, ns2, xv), r2, y0);
            const uint64_t q = f2_fma(f2_fma(y1, ns2, xv), r2, y1);
            x[i] = f2_lo(q);
            x[i + 1] = f2_hi(q);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = __fdiv_rn(x[i], s);
    }
}

// Quantising append: bf16 K/V rows of new tokens into an FP8 E4M3 cache
// ("attention kernels", "what to check": FP8 KV).  Each element is divided by
// its KV head's fp32 scale (the IEEE quotient, div_by_scale8) and rounded to
// E4M3.  One CTA per new token, as kv_append_kernel; a thread turns a chunk
// of 8 bf16 (16 bytes) into 8 bytes.
__global__ void __launch_bounds__(kAppendThreads)
kv_append_quant_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                       const int64_t *__restrict__ slots, uint2 *k_cache, uint2 *v_cache,
                       const float *__restrict__ k_scale, const float *__restrict__ v_scale,
                       int32_t hkv, int32_t row_vec, int32_t lg_cp, int32_t lg_bs,
                       int64_t pool_slots, uint32_t *flags) {
    const int t = blockIdx.x;
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) return;
    if (slot >= pool_slots) {
        if (threadIdx.x == 0) raise_flag(flags, kFlagSlot);
        return;
    }
    const int64_t blk = slot >> lg_bs, off = slot & ((1 << lg_bs) - 1);
    const int n = hkv << lg_cp;
    for (int i = threadIdx.x; i < n; i += kAppendThreads) {
        const int h = i >> lg_cp, c = i & ((1 << lg_cp) - 1);
        const bool isk = c < row_vec;
        const int ch = isk ? c : c - row_vec;
        const int64_t src = (static_cast<int64_t>(t) * hkv + h) * row_vec + ch;   // in uint4
        const int64_t dst = (((blk * hkv + h) << lg_bs) + off) * row_vec + ch;    // in uint2
        const float s = __ldg((isk ? k_scale : v_scale) + h);
        const uint4 x = __ldg((isk ? k_new : v_new) + src);
        const uint32_t in[4] = {x.x, x.y, x.z, x.w};
        float v[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = unpack_bf16x2(in[k]);
            v[2 * k] = f.x;
            v[2 * k + 1] = f.y;
        }
        div_by_scale8(v, s, __frcp_rn(s));
        uint32_t b[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) b[k] = f32x2_to_e4m3x2(v[2 * k], v[2 * k + 1]);
        (isk ? k_cache : v_cache)[dst] = make_uint2(b[0] | (b[1] << 16), b[2] | (b[3] << 16));
    }
}

cudaError_t launch_kv_append_quant(const void *k_new, const void *v_new, const int64_t *slots,
                                   int32_t num_tokens, void *k_cache, void *v_cache,
                                   const float *k_scale, const float *v_scale, int32_t hkv,
                                   int32_t head_dim, int32_t block_size, int64_t pool_slots,
                                   uint32_t *flags, cudaStream_t stream) {
    const int row_vec = head_dim / 8;
    const int lg_cp = lg2_exact(2 * row_vec), lg_bs = lg2_exact(block_size);
    if (lg_cp < 0 || lg_bs < 0 || (static_cast<long long>(hkv) << lg_cp) > (1LL << 30))
        return cudaErrorInvalidValue;
    if (num_tokens == 0) return cudaSuccess;
    kv_append_quant_kernel<<<static_cast<unsigned>(num_tokens), kAppendThreads, 0, stream>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new), slots,
        static_cast<uint2 *>(k_cache), static_cast<uint2 *>(v_cache), k_scale, v_scale, hkv,
        row_vec, lg_cp, lg_bs, pool_slots, flags);
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
