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
// the bulk kernel (2-64 ranks, every buffer at one 16-byte phase on element
// boundaries; the two-shot's first shot up to 16 ranks); bulk_scatter_eligible:
// a reduce-scatter can (2-16 ranks, the inputs at one phase);
// bulk_tree_eligible: a tree-order one-shot can (2-8, 12 and 16 ranks, every
// buffer at one 16-byte phase).  The launchers use their own tiling.
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

// The one-shot, the reduce-scatter, the bf16-wire one-shot and the
// tree-order one-shot over rank buffers at different 16-byte phases
// (rr_mixed.cu): every rank's tile staged
// at its own shift, whole-vector stores to every output at its own phase.
// mixed_eligible: a plain call of 2-64 ranks on element boundaries.
bool mixed_eligible(const RankParams& p, int esize);
template <class Ty, int OP>
cudaError_t launch_oneshot_mixed(const RankParams& p, cudaStream_t s);
template <class Ty, int OP>
cudaError_t launch_scatter_mixed(const RankParams& p, cudaStream_t s);
cudaError_t launch_oneshot_wire_mixed(int op, const RankParams& p, cudaStream_t s);
// the tree-order one-shot the same way (2-16 ranks; the whole buffer is one segment)
bool mixed_tree_eligible(const RankParams& p, int esize);
template <class Ty, int OP>
cudaError_t launch_tree_mixed(const RankParams& p, cudaStream_t s);

// The tree's pairwise order ([P3] section 6: ranks pair up, pairs pair up,
// log2 N levels) folded per element in registers.  Ranks are pushed in order
// 0..N-1 onto a stack of partial blocks: pushing rank j combines it with the
// blocks it completes (one per trailing one bit of j, earlier block on the
// left), so slot[b] always holds a block of 2^b ranks.  At the end the blocks
// for the set bits of N are combined from the smallest upwards, each larger
// (earlier) block on the left: exactly the level schedule in which a rank
// without a partner carries its value up.
template <class Ty, int OP, int W, int NMAX>
__device__ __forceinline__ void tree_fold_lanes(const RankParams& p, uint64_t e0, bool vec)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    constexpr int LV = NMAX <= 2 ? 2 : (NMAX <= 4 ? 3 : (NMAX <= 8 ? 4 : 7));  // log2(NMAX) + 1
    Acc slot[LV][W];
    Acc cur[W];
    const int n = p.n;
#pragma unroll
    for (int g = 0; g < NMAX; g += kGroup) {
        if (g < n) {
            Acc v[kGroup][W];
#pragma unroll
            for (int k = 0; k < kGroup; ++k) {
                if (g + k < n && g + k < NMAX) {
                    const T* src = static_cast<const T*>(p.in[g + k]) + e0;
                    if constexpr (W == Ty::L) {
                        if (vec) {
                            Ty::unpack(ldv(src), v[k]);
                            continue;
                        }
                    }
                    v[k][0] = Ty::ld1(src);
                }
            }
#pragma unroll
            for (int k = 0; k < kGroup; ++k) {
                const int j = g + k;
                if (j < n && j < NMAX) {
#pragma unroll
                    for (int l = 0; l < W; ++l) cur[l] = v[k][l];
                    int lvl = 0;
#pragma unroll
                    for (int b = 0; b < LV - 1; ++b) {
                        if (((j >> b) & 1) && lvl == b) {
#pragma unroll
                            for (int l = 0; l < W; ++l) cur[l] = apply<OP>(slot[b][l], cur[l]);
                            lvl = b + 1;
                        }
                    }
#pragma unroll
                    for (int b = 0; b < LV; ++b)
                        if (b == lvl)
#pragma unroll
                            for (int l = 0; l < W; ++l) slot[b][l] = cur[l];
                }
            }
        }
    }
    bool have = false;
#pragma unroll
    for (int b = 0; b < LV; ++b) {
        if ((n >> b) & 1) {
#pragma unroll
            for (int l = 0; l < W; ++l) cur[l] = have ? apply<OP>(slot[b][l], cur[l]) : slot[b][l];
            have = true;
        }
    }
#pragma unroll
    for (int l = 0; l < W; ++l) cur[l] = finish<OP>(cur[l], p.divisor);
    if constexpr (W == Ty::L) {
        if (vec) {
            const uint4 r = Ty::pack(cur);
#pragma unroll 4
            for (int o = 0; o < n; ++o) stv(static_cast<T*>(p.out[o]) + e0, r);
            return;
        }
    }
    for (int o = 0; o < n; ++o) Ty::st1(static_cast<T*>(p.out[o]) + e0, cur[0]);
}

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
