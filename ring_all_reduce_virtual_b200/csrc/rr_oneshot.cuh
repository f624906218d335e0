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

// The bulk-copy kernels (rr_bulk.cuh; rr_bulk.cu, rr_bulk_rs.cu,
// rr_bulk_tree.cu).  bulk_eligible: a one-shot call in ring order can take
// the bulk kernel (rank count 2, 4, 8, 16, 32 or 64; 16-byte aligned buffers
// and chunks; a plain call over whole chunks); bulk_scatter_eligible: a
// reduce-scatter can (2-16 ranks, parts of whole vectors);
// bulk_tree_eligible: a tree-order one-shot can (2-16 ranks, a buffer of
// whole vectors).  The launchers use their own tiling.
bool bulk_eligible(const RankParams& p, int esize);
bool bulk_scatter_eligible(const RankParams& p, int esize);
bool bulk_tree_eligible(const RankParams& p, int esize);
template <class Ty, int OP>
cudaError_t launch_oneshot_bulk(const RankParams& p, cudaStream_t s);
template <class Ty, int OP>
cudaError_t launch_scatter_bulk(const RankParams& p, cudaStream_t s);
template <class Ty, int OP>
cudaError_t launch_tree_bulk(const RankParams& p, cudaStream_t s);
cudaError_t launch_oneshot_wire_bulk(int op, const RankParams& p, cudaStream_t s);

#define RR_FOR_EACH_TYPE_OP(X)                                                                   \
    X(F32T, kSum) X(F32T, kAvg) X(F32T, kMax) X(F32T, kMin) X(F32T, kProd) X(BF16T, kSum)         \
    X(BF16T, kAvg) X(BF16T, kMax) X(BF16T, kMin) X(BF16T, kProd) X(I32T, kSum) X(I32T, kMax)     \
    X(I32T, kMin) X(I32T, kProd) X(F16T, kSum) X(F16T, kAvg) X(F16T, kMax) X(F16T, kMin)         \
    X(F16T, kProd)

#define RR_DECLARE_ONESHOT(TY, OP)                                                               \
    extern template cudaError_t launch_oneshot_ring<TY, OP>(const RankParams&, uint64_t, cudaStream_t); \
    extern template cudaError_t launch_oneshot_tree<TY, OP>(const RankParams&, uint64_t, cudaStream_t); \
    extern template cudaError_t launch_oneshot_bulk<TY, OP>(const RankParams&, cudaStream_t); \
    extern template cudaError_t launch_scatter_bulk<TY, OP>(const RankParams&, cudaStream_t); \
    extern template cudaError_t launch_tree_bulk<TY, OP>(const RankParams&, cudaStream_t);
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
template <>
inline cudaError_t launch_scatter_bulk<I32T, kAvg>(const RankParams&, cudaStream_t)
{
    return cudaErrorInvalidValue;
}
template <>
inline cudaError_t launch_tree_bulk<I32T, kAvg>(const RankParams&, cudaStream_t)
{
    return cudaErrorInvalidValue;
}

}  // namespace rr
