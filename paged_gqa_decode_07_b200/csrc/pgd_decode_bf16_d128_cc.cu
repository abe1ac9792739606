// Decode variants with CUDA-core math (FMA dot products, warp-shuffle sums):
// head_dim 128, bf16 KV cache, block_size 16/32/64, up to 4 or 8 query rows.
// Kept to compare with the tensor-core variants (pgd_set_decode_math).
#include "pgd_decode_family.cuh"

namespace pgd {
PGD_INSTANTIATE_CUDA_CORE(4)
PGD_INSTANTIATE_CUDA_CORE(8)
}  // namespace pgd
