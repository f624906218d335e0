// rr_tree.cu -- the one-shot all-reduce in the tree's pairwise order.
//
// Sources: [P3] "Training gradient sync and collective communication"
// (geek-doc.cn), section 6 (tree reduction: ranks pair up, pairs pair up,
// log2 N levels).
#include "rr_oneshot.cuh"

namespace rr {

namespace {

// ------------------------------------------------ one-shot, tree order
// tree_fold_lanes (rr_oneshot.cuh) folds one element or one vector per
// thread; tree_vectors below keeps several vectors in flight.

// For N <= NMAX <= 8: every rank's vectors for VPT vectors are loaded first
// (N * VPT loads in flight per thread), then each vector is folded in tree
// order with the same stack as tree_fold_lanes, levels fixed at compile time.
template <class Ty, int OP, int NMAX, int VPT, bool EXACT>
__device__ __forceinline__ void tree_vectors(const RankParams& p, uint64_t v0, uint64_t nv, uint64_t head)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;
    constexpr int LV = NMAX <= 2 ? 2 : (NMAX <= 4 ? 3 : 4);  // log2(NMAX) + 1 stack levels
    const int n = EXACT ? NMAX : p.n;
    uint64_t off[VPT];
    bool ok[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        const uint64_t v = v0 + (uint64_t)u * kThreads + threadIdx.x;
        ok[u] = v < nv;
        off[u] = head + v * L;
    }
    uint4 raw[NMAX][VPT];
#pragma unroll
    for (int j = 0; j < NMAX; ++j)
        if (j < n) {
            const T* src = static_cast<const T*>(p.in[j]);
#pragma unroll
            for (int u = 0; u < VPT; ++u)
                if (ok[u]) raw[j][u] = ldv(src + off[u]);
        }
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        if (!ok[u]) continue;
        Acc slot[LV][L];
        Acc cur[L];
#pragma unroll
        for (int j = 0; j < NMAX; ++j) {
            if (j < n) {
                Ty::unpack(raw[j][u], cur);
                int lvl = 0;
#pragma unroll
                for (int b = 0; b < LV - 1; ++b) {
                    if (((j >> b) & 1) && lvl == b) {
#pragma unroll
                        for (int l = 0; l < L; ++l) cur[l] = apply<OP>(slot[b][l], cur[l]);
                        lvl = b + 1;
                    }
                }
#pragma unroll
                for (int b = 0; b < LV; ++b)
                    if (b == lvl)
#pragma unroll
                        for (int l = 0; l < L; ++l) slot[b][l] = cur[l];
            }
        }
        bool have = false;
#pragma unroll
        for (int b = 0; b < LV; ++b) {
            if ((n >> b) & 1) {
#pragma unroll
                for (int l = 0; l < L; ++l) cur[l] = have ? apply<OP>(slot[b][l], cur[l]) : slot[b][l];
                have = true;
            }
        }
#pragma unroll
        for (int l = 0; l < L; ++l) cur[l] = finish<OP>(cur[l], p.divisor);
        const uint4 r = Ty::pack(cur);
#pragma unroll 4
        for (int o = 0; o < n; ++o) stv(static_cast<T*>(p.out[o]) + off[u], r);
    }
}

template <class Ty, int OP, int NMAX, int VPT, bool EXACT>
__global__ void __launch_bounds__(kThreads) oneshot_tree_kernel(const __grid_constant__ RankParams p)
{
    constexpr int L = Ty::L;
    constexpr uint64_t TE = (uint64_t)kThreads * VPT * L;
    const int tid = threadIdx.x;
    const int ph = p.vec_ok ? phase_of(static_cast<const typename Ty::T*>(p.in[0]), L) : -1;
    uint64_t head = 0, nv = 0;
    if (ph >= 0) {
        head = (uint64_t)((L - ph) & (L - 1));
        if (head > p.count) head = p.count;
        nv = (p.count - head) / L;
    }
    const uint64_t tail_lo = head + nv * L;
    for (uint64_t tile = blockIdx.x; tile < p.tps; tile += gridDim.x) {
        if (ph < 0) {
            for (int k = 0; k < (int)(TE / kThreads); ++k) {
                const uint64_t e = tile * TE + (uint64_t)k * kThreads + tid;
                if (e < p.count) tree_fold_lanes<Ty, OP, 1, NMAX>(p, e, false);
            }
            continue;
        }
        if (tile == 0 && (uint64_t)tid < head + (p.count - tail_lo)) {
            const uint64_t e = (uint64_t)tid < head ? (uint64_t)tid : tail_lo + ((uint64_t)tid - head);
            tree_fold_lanes<Ty, OP, 1, NMAX>(p, e, false);
        }
        if constexpr (NMAX <= 8) {
            tree_vectors<Ty, OP, NMAX, VPT, EXACT>(p, tile * (TE / L), nv, head);
        } else {
            for (int u = 0; u < VPT; ++u) {
                const uint64_t v = tile * (TE / L) + (uint64_t)u * kThreads + tid;
                if (v < nv) tree_fold_lanes<Ty, OP, L, NMAX>(p, head + v * L, true);
            }
        }
    }
}

}  // namespace

template <class Ty, int OP>
cudaError_t launch_oneshot_tree(const RankParams& p, uint64_t work, cudaStream_t s)
{
    if (bulk_tree_eligible(p, (int)sizeof(typename Ty::T))) return launch_tree_bulk<Ty, OP>(p, s);
    if (!p.vec_ok && mixed_tree_eligible(p, (int)sizeof(typename Ty::T))) return launch_tree_mixed<Ty, OP>(p, s);
    const int n = p.n;
    constexpr int V = kVptReduce;
    switch (n) {
    case 2: return launch_all(oneshot_tree_kernel<Ty, OP, 2, V, true>, p, work, s);
    case 4: return launch_all(oneshot_tree_kernel<Ty, OP, 4, V, true>, p, work, s);
    case 8: return launch_all(oneshot_tree_kernel<Ty, OP, 8, V, true>, p, work, s);
    }
    if (n <= 4) return launch_all(oneshot_tree_kernel<Ty, OP, 4, V, false>, p, work, s);
    if (n <= 8) return launch_all(oneshot_tree_kernel<Ty, OP, 8, V, false>, p, work, s);
    return launch_all(oneshot_tree_kernel<Ty, OP, kMaxRanks, V, false>, p, work, s);
}

#define RR_INSTANTIATE(TY, OP) \
    template cudaError_t launch_oneshot_tree<TY, OP>(const RankParams&, uint64_t, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_INSTANTIATE)
#undef RR_INSTANTIATE

}  // namespace rr
