// rr_oneshot.cuh -- launchers of the one-shot kernels (ring order and tree
// order), compiled in their own files (rr_oneshot.cu, rr_tree.cu) and
// instantiated there for every (element type, op) pair.
#pragma once

#include "rr_launch.cuh"

namespace rr {

template <class Ty, int OP>
cudaError_t launch_oneshot_ring(const RankParams& p, uint64_t work, cudaStream_t s);
template <class Ty, int OP>
cudaError_t launch_oneshot_tree(const RankParams& p, uint64_t work, cudaStream_t s);

// The bulk-copy one-shot (rr_bulk.cu): bulk_eligible says whether a one-shot
// call can take it (rank count 2, 4, 8, 16, 32 or 64; 16-byte aligned buffers and
// chunks; a plain call over whole chunks), launch_oneshot_bulk launches it
// with its own tiling.
bool bulk_eligible(const RankParams& p, int esize);
template <class Ty, int OP>
cudaError_t launch_oneshot_bulk(const RankParams& p, cudaStream_t s);

#define RR_FOR_EACH_TYPE_OP(X)                                                                   \
    X(F32T, kSum) X(F32T, kAvg) X(F32T, kMax) X(F32T, kMin) X(F32T, kProd) X(BF16T, kSum)         \
    X(BF16T, kAvg) X(BF16T, kMax) X(BF16T, kMin) X(BF16T, kProd) X(I32T, kSum) X(I32T, kMax)     \
    X(I32T, kMin) X(I32T, kProd) X(F16T, kSum) X(F16T, kAvg) X(F16T, kMax) X(F16T, kMin)         \
    X(F16T, kProd)

#define RR_DECLARE_ONESHOT(TY, OP)                                                               \
    extern template cudaError_t launch_oneshot_ring<TY, OP>(const RankParams&, uint64_t, cudaStream_t); \
    extern template cudaError_t launch_oneshot_tree<TY, OP>(const RankParams&, uint64_t, cudaStream_t); \
    extern template cudaError_t launch_oneshot_bulk<TY, OP>(const RankParams&, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_DECLARE_ONESHOT)
#undef RR_DECLARE_ONESHOT

// I32T has no AVG; these are never launched (the host rejects AVG on int32).
template <>
inline cudaError_t launch_oneshot_ring<I32T, kAvg>(const RankParams&, uint64_t, cudaStream_t)
{
    return cudaErrorInvalidValue;
}
template <>
inline cudaError_t launch_oneshot_tree<I32T, kAvg>(const RankParams&, uint64_t, cudaStream_t)
{
    return cudaErrorInvalidValue;
}
template <>
inline cudaError_t launch_oneshot_bulk<I32T, kAvg>(const RankParams&, cudaStream_t)
{
    return cudaErrorInvalidValue;
}

}  // namespace rr
