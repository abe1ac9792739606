// pgd_decode_family.cuh -- definitions of the per-variant launchers; each
// pgd_decode_*.cu unit includes this and instantiates one family.
#pragma once

#include <atomic>

#include "pgd_launch.h"

namespace pgd {

template <int D, int BS, int NT, bool FP8, int CC = 0>
static void *decode_kernel_ptr() {
    constexpr int NS = Stages<D, FP8>::value;
    return reinterpret_cast<void *>(&paged_decode_kernel<D, BS, NT, FP8, NS, CC>);
}

template <int D, int BS, int NT, bool FP8, int CC = 0>
static cudaError_t ensure_smem_attr() {
    constexpr int NS = Stages<D, FP8>::value;
    using C = DecodeCfg<D, BS, NT, FP8, NS, CC>;
    static std::atomic<uint64_t> done_mask{0};   // one bit per device ordinal < 64
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const uint64_t bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done_mask.load() & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(decode_kernel_ptr<D, BS, NT, FP8, CC>(),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e == cudaSuccess && bit) done_mask.fetch_or(bit);
    return e;
}

template <int D, int BS, int NT, bool FP8, int CC>
cudaError_t launch_decode(const DecodeLaunchArgs &a) {
    constexpr int NS = Stages<D, FP8>::value;
    using C = DecodeCfg<D, BS, NT, FP8, NS, CC>;
    cudaError_t e = ensure_smem_attr<D, BS, NT, FP8, CC>();
    if (e != cudaSuccess) return e;
    // programmatic dependent launch: the kernel waits (griddepcontrol.wait)
    // for the previous work on the stream before its first global read
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(a.grid));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, paged_decode_kernel<D, BS, NT, FP8, NS, CC>, a.tmK, a.tmV,
                              a.p);
}

template <int D, int BS, int NT, bool FP8, int CC>
int decode_ctas_per_sm() {
    constexpr int NS = Stages<D, FP8>::value;
    using C = DecodeCfg<D, BS, NT, FP8, NS, CC>;
    if (ensure_smem_attr<D, BS, NT, FP8, CC>() != cudaSuccess) return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel_ptr<D, BS, NT, FP8, CC>(),
                                                      kThreads, C::SMEM) != cudaSuccess)
        return 0;
    return n;
}

#define PGD_INSTANTIATE_FAMILY(D, FP8)                                          \
    template cudaError_t launch_decode<D, 16, 1, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 32, 1, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 64, 1, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 16, 2, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 32, 2, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 64, 2, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 16, 4, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 32, 4, FP8>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<D, 64, 4, FP8>(const DecodeLaunchArgs &); \
    template int decode_ctas_per_sm<D, 16, 1, FP8>();                           \
    template int decode_ctas_per_sm<D, 32, 1, FP8>();                           \
    template int decode_ctas_per_sm<D, 64, 1, FP8>();                           \
    template int decode_ctas_per_sm<D, 16, 2, FP8>();                           \
    template int decode_ctas_per_sm<D, 32, 2, FP8>();                           \
    template int decode_ctas_per_sm<D, 64, 2, FP8>();                           \
    template int decode_ctas_per_sm<D, 16, 4, FP8>();                           \
    template int decode_ctas_per_sm<D, 32, 4, FP8>();                           \
    template int decode_ctas_per_sm<D, 64, 4, FP8>();

// CUDA-core comparison variants (bf16, head_dim 128, up to CC query rows)
#define PGD_INSTANTIATE_CUDA_CORE(CC)                                             \
    template cudaError_t launch_decode<128, 16, 1, false, CC>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<128, 32, 1, false, CC>(const DecodeLaunchArgs &); \
    template cudaError_t launch_decode<128, 64, 1, false, CC>(const DecodeLaunchArgs &); \
    template int decode_ctas_per_sm<128, 16, 1, false, CC>();                           \
    template int decode_ctas_per_sm<128, 32, 1, false, CC>();                           \
    template int decode_ctas_per_sm<128, 64, 1, false, CC>();

}  // namespace pgd
