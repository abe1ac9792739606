// pgd_launch.h -- host-side declarations shared by the C ABI and the kernel
// translation units (one unit per compiled family of decode variants).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pgd_decode.cuh"

namespace pgd {

struct DecodeLaunchArgs {
    DecodeParams p;
    CUtensorMap tmK, tmV;
    int grid;
    cudaStream_t stream;
};

// Shared-memory pipeline depth per family: 96 KB of K/V stages per CTA for
// head_dim 128 (two CTAs per SM), 192 KB for head_dim 256 (one per SM).
template <int D, bool FP8>
struct Stages {
    static constexpr int value = FP8 ? 6 : 3;
};

// CC = 0: tensor-core consumers; CC = 4 / 8: the CUDA-core comparison variant
template <int D, int BS, int NT, bool FP8, int CC = 0>
cudaError_t launch_decode(const DecodeLaunchArgs &a);

// Resident CTAs per SM for this variant (0 if it cannot launch).
template <int D, int BS, int NT, bool FP8, int CC = 0>
int decode_ctas_per_sm();

#define PGD_DECLARE_FAMILY(D, FP8)                                                    \
    extern template cudaError_t launch_decode<D, 16, 1, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 32, 1, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 64, 1, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 16, 2, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 32, 2, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 64, 2, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 16, 4, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 32, 4, FP8>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<D, 64, 4, FP8>(const DecodeLaunchArgs &); \
    extern template int decode_ctas_per_sm<D, 16, 1, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 32, 1, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 64, 1, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 16, 2, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 32, 2, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 64, 2, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 16, 4, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 32, 4, FP8>();                           \
    extern template int decode_ctas_per_sm<D, 64, 4, FP8>();

PGD_DECLARE_FAMILY(128, false)
PGD_DECLARE_FAMILY(256, false)
PGD_DECLARE_FAMILY(128, true)

#define PGD_DECLARE_CUDA_CORE(CC)                                                         \
    extern template cudaError_t launch_decode<128, 16, 1, false, CC>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<128, 32, 1, false, CC>(const DecodeLaunchArgs &); \
    extern template cudaError_t launch_decode<128, 64, 1, false, CC>(const DecodeLaunchArgs &); \
    extern template int decode_ctas_per_sm<128, 16, 1, false, CC>();                           \
    extern template int decode_ctas_per_sm<128, 32, 1, false, CC>();                           \
    extern template int decode_ctas_per_sm<128, 64, 1, false, CC>();

PGD_DECLARE_CUDA_CORE(4)
PGD_DECLARE_CUDA_CORE(8)

// kv_append and the standalone LSE merge (pgd_aux.cu)
cudaError_t launch_kv_append(const void *k_new, const void *v_new, const int64_t *slots,
                             int32_t num_tokens, void *k_cache, void *v_cache, int32_t hkv,
                             int32_t row_bytes, int32_t block_size, int64_t pool_slots,
                             uint32_t *flags, cudaStream_t stream);

cudaError_t launch_kv_append_quant(const void *k_new, const void *v_new, const int64_t *slots,
                                   int32_t num_tokens, void *k_cache, void *v_cache,
                                   const float *k_scale, const float *v_scale, int32_t hkv,
                                   int32_t head_dim, int32_t block_size, int64_t pool_slots,
                                   uint32_t *flags, cudaStream_t stream);

cudaError_t launch_merge_partials(const float *o_part, const float *lse_part, int32_t parts,
                                  int32_t rows, int32_t head_dim, uint16_t *out, float *lse_out,
                                  cudaStream_t stream);

}  // namespace pgd
