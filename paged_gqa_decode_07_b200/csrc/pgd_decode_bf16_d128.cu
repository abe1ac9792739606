// Decode variants: head_dim 128, bf16 KV cache, block_size 16/32/64, group <= 8 / 16.
#include "pgd_decode_family.cuh"

namespace pgd {
PGD_INSTANTIATE_FAMILY(128, false)
}  // namespace pgd
