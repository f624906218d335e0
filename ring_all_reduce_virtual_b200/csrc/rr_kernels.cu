// rr_kernels.cu -- the collectives' kernels and their launchers.
//
// All kernels are HBM-bound streaming kernels: each input byte is read once
// and each output byte written once per launch, with 128-bit vector access
// and a grid-stride loop over (segment, tile) work items sized to one wave of
// resident CTAs.  No kernel waits on another CTA or another launch.
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "The five primitives", "Ring all-reduce and communication volume"
// and "alpha-beta model"; [P3] "Training gradient sync and collective
// communication" (geek-doc.cn), sections 3 and 6.
#include <type_traits>

#include "rr_device.cuh"
#include "rr_internal.h"

namespace rr {

namespace {


// ------------------------------------------------ one-shot, ring order
// Segment c = chunk c of every rank buffer; its fold starts on rank c and
// walks the ring (c, c+1, ..., c+N-1 mod N); the result goes to all N
// buffers.  One launch replaces the ring's 2(N-1) steps with the same bits.
template <class Ty, int OP, int VPT, int G>
__global__ void __launch_bounds__(kThreads) oneshot_ring_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t total = p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t c = w / p.tps, tile = w - c * p.tps;
        // chunk c clipped to this launch's element range
        const uint64_t c_lo = c * p.C, c_hi = c_lo + p.C < p.count ? c_lo + p.C : p.count;
        const uint64_t lo = c_lo > p.lo ? c_lo : p.lo;
        const uint64_t hi = c_hi < p.hi ? c_hi : p.hi;
        if (lo >= hi) continue;
        const uint64_t len = hi - lo;
        const int start = (int)c;
        auto in = [&](int j) {
            int r = start + j;
            if (r >= p.n) r -= p.n;
            return static_cast<const T*>(p.in[r]) + lo;
        };
        auto out = [&](int o) { return static_cast<T*>(p.out[p.owner_only ? start : o]) + lo; };
        fold_tile<Ty, OP, VPT, G>(in, p.n, out, p.owner_only ? 1 : p.n, len, tile, p.vec_ok, p.divisor);
    }
}

// ------------------------------------------------- chunk broadcast
// Two-shot's second shot: segment c = chunk c, read once from its owner
// (rank c) and written to chunk c of the N-1 other ranks.
template <class Ty>
__global__ void __launch_bounds__(kThreads) chunk_bcast_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t total = p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t c = w / p.tps, tile = w - c * p.tps;
        const uint64_t lo = c * p.C;
        if (lo >= p.count) continue;
        const uint64_t len = p.count - lo < p.C ? p.count - lo : p.C;
        const int owner = (int)c;
        auto in = [&](int) { return static_cast<const T*>(p.in[owner]) + lo; };
        auto out = [&](int o) { return static_cast<T*>(p.out[o < owner ? o : o + 1]) + lo; };
        fold_tile<Ty, kSum, kVptMove, 1>(in, 1, out, p.n - 1, len, tile, p.vec_ok, 1.0f);
    }
}

// -------------------------------------------------- reduce-scatter
// Segment r = part r: fold of in_{r}, in_{r+1}, ... (ring order of chunk r)
// at offset r*C, written to out_r.
template <class Ty, int OP, int VPT, int G>
__global__ void __launch_bounds__(kThreads) reduce_scatter_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t total = p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t r = w / p.tps, tile = w - r * p.tps;
        const uint64_t lo = r * p.C;
        const int start = (int)r;
        auto in = [&](int j) {
            int q = start + j;
            if (q >= p.n) q -= p.n;
            return static_cast<const T*>(p.in[q]) + lo;
        };
        auto out = [&](int) { return static_cast<T*>(p.out[start]); };
        fold_tile<Ty, OP, VPT, G>(in, p.n, out, 1, p.C, tile, p.vec_ok, p.divisor);
    }
}

// ------------------------------------------------------ all-gather
// Segment q = rank q's part: read once, written to offset q*C of every
// output.
template <class Ty>
__global__ void __launch_bounds__(kThreads) all_gather_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t total = p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t q = w / p.tps, tile = w - q * p.tps;
        auto in = [&](int) { return static_cast<const T*>(p.in[q]); };
        auto out = [&](int o) { return static_cast<T*>(p.out[o]) + q * p.C; };
        fold_tile<Ty, kSum, kVptMove, 1>(in, 1, out, p.n, p.C, tile, p.vec_ok, 1.0f);
    }
}

// ------------------------------------------------------ all-to-all
// Segment (r, q): block r of rank q goes to block q of rank r.
template <class Ty>
__global__ void __launch_bounds__(kThreads) all_to_all_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t total = p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t s = w / p.tps, tile = w - s * p.tps;
        const uint64_t r = s / (uint64_t)p.n, q = s - r * (uint64_t)p.n;
        auto in = [&](int) { return static_cast<const T*>(p.in[q]) + r * p.C; };
        auto out = [&](int) { return static_cast<T*>(p.out[r]) + q * p.C; };
        fold_tile<Ty, kSum, kVptMove, 1>(in, 1, out, 1, p.C, tile, 1, 1.0f);
    }
}

// ------------------------------------------------ one-shot, tree order
// The tree's pairwise order ([P3] section 6: ranks pair up, pairs pair up,
// log2 N levels) folded per element in registers.  Ranks are pushed in order
// 0..N-1 onto a stack of partial blocks: pushing rank j combines it with the
// blocks it completes (one per trailing one bit of j, earlier block on the
// left), so slot[b] always holds a block of 2^b ranks.  At the end the blocks
// for the set bits of N are combined from the smallest upwards, each larger
// (earlier) block on the left: exactly the level schedule in which a rank
// without a partner carries its value up.
template <class Ty, int OP, int W>
__device__ __forceinline__ void tree_fold_lanes(const RankParams& p, uint64_t e0, bool vec)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    Acc slot[7][W];
    Acc cur[W];
    const int n = p.n;
#pragma unroll
    for (int g = 0; g < kMaxRanks; g += kGroup) {
        if (g < n) {
            Acc v[kGroup][W];
#pragma unroll
            for (int k = 0; k < kGroup; ++k) {
                if (g + k < n) {
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
                if (j < n) {
#pragma unroll
                    for (int l = 0; l < W; ++l) cur[l] = v[k][l];
                    int lvl = 0;
#pragma unroll
                    for (int b = 0; b < 6; ++b) {
                        if (((j >> b) & 1) && lvl == b) {
#pragma unroll
                            for (int l = 0; l < W; ++l) cur[l] = apply<OP>(slot[b][l], cur[l]);
                            lvl = b + 1;
                        }
                    }
#pragma unroll
                    for (int b = 0; b < 7; ++b)
                        if (b == lvl)
#pragma unroll
                            for (int l = 0; l < W; ++l) slot[b][l] = cur[l];
                }
            }
        }
    }
    bool have = false;
#pragma unroll
    for (int b = 0; b < 7; ++b) {
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

// For N <= NMAX <= 8: every rank's vectors for VPT vectors are loaded first
// (N * VPT loads in flight per thread), then each vector is folded in tree
// order with the same stack as tree_fold_lanes, levels fixed at compile time.
template <class Ty, int OP, int NMAX, int VPT>
__device__ __forceinline__ void tree_vectors(const RankParams& p, uint64_t v0, uint64_t nv, uint64_t head)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;
    constexpr int LV = NMAX <= 2 ? 2 : (NMAX <= 4 ? 3 : 4);  // log2(NMAX) + 1 stack levels
    const int n = p.n;
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

template <class Ty, int OP, int NMAX, int VPT>
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
                if (e < p.count) tree_fold_lanes<Ty, OP, 1>(p, e, false);
            }
            continue;
        }
        if (tile == 0 && (uint64_t)tid < head + (p.count - tail_lo)) {
            const uint64_t e = (uint64_t)tid < head ? (uint64_t)tid : tail_lo + ((uint64_t)tid - head);
            tree_fold_lanes<Ty, OP, 1>(p, e, false);
        }
        if constexpr (NMAX <= 8) {
            tree_vectors<Ty, OP, NMAX, VPT>(p, tile * (TE / L), nv, head);
        } else {
            for (int u = 0; u < VPT; ++u) {
                const uint64_t v = tile * (TE / L) + (uint64_t)u * kThreads + tid;
                if (v < nv) tree_fold_lanes<Ty, OP, L>(p, head + v * L, true);
            }
        }
    }
}

// ------------------------------------------------------- table steps
// One ring step or one tree level: every segment folds in0 op in1 into out
// (nin == 2) or copies in0 to out (nin == 1).
template <class Ty, int OP>
__global__ void __launch_bounds__(kThreads) step_kernel(const __grid_constant__ StepParams p)
{
    using T = typename Ty::T;
    const uint64_t total = (uint64_t)p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t s = w / p.tps, tile = w - s * p.tps;
        const StepSeg& sg = p.seg[s];
        if (sg.len == 0) continue;
        auto in = [&](int j) { return static_cast<const T*>(j == 0 ? sg.in0 : sg.in1); };
        auto out = [&](int) { return static_cast<T*>(sg.out); };
        fold_tile<Ty, OP, kVptMove, 1>(in, p.nin, out, 1, sg.len, tile, p.vec_ok, p.divisor);
    }
}

// ------------------------------------------------------------ launching

// One CTA per work item, up to the grid limit.  (A grid of one wave of
// resident CTAs looping over the tiles measured about 15 % slower on the
// 8 x 256 MiB all-reduce.)
template <class P>
cudaError_t launch_all(void (*kernel)(P), const P& p, uint64_t work, cudaStream_t s)
{
    if (work == 0) return cudaSuccess;
    const uint64_t grid = work < kMaxGrid ? work : kMaxGrid;
    kernel<<<(unsigned)grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <class F>
cudaError_t with_type(int dtype, int op, F&& f)
{
    auto by_op = [&]<class Ty>() -> cudaError_t {
        switch (op) {
        case kSum: return f.template operator()<Ty, kSum>();
        case kMax: return f.template operator()<Ty, kMax>();
        case kMin: return f.template operator()<Ty, kMin>();
        case kProd: return f.template operator()<Ty, kProd>();
        case kAvg:
            if constexpr (std::is_same_v<Ty, I32T>) return cudaErrorInvalidValue;
            else return f.template operator()<Ty, kAvg>();
        }
        return cudaErrorInvalidValue;
    };
    switch (dtype) {
    case kF32: return by_op.template operator()<F32T>();
    case kBF16: return by_op.template operator()<BF16T>();
    case kI32: return by_op.template operator()<I32T>();
    }
    return cudaErrorInvalidValue;
}

}  // namespace

uint64_t tile_elems(int dtype, int vpt)
{
    return (uint64_t)kThreads * (uint64_t)vpt * (dtype == kBF16 ? 8u : 4u);
}

cudaError_t launch_rank_kernel(int kind, int dtype, int op, const RankParams& p, cudaStream_t s)
{
    const uint64_t work = kind == kOneshotTree ? p.tps : p.nseg * p.tps;
    if (kind == kAllGather || kind == kAllToAll || kind == kChunkBroadcast) op = kSum;
    const int vpt = reduce_vpt(p.n);
    return with_type(dtype, op, [&]<class Ty, int OP>() -> cudaError_t {
        switch (kind) {
        case kOneshotRing:
            if (vpt == 8) return launch_all(oneshot_ring_kernel<Ty, OP, 8, 1>, p, work, s);
            if (vpt == 4) return launch_all(oneshot_ring_kernel<Ty, OP, 4, 3>, p, work, s);
            return launch_all(oneshot_ring_kernel<Ty, OP, kVptReduce, kGroup>, p, work, s);
        case kReduceScatter:
            if (vpt == 8) return launch_all(reduce_scatter_kernel<Ty, OP, 8, 1>, p, work, s);
            if (vpt == 4) return launch_all(reduce_scatter_kernel<Ty, OP, 4, 3>, p, work, s);
            return launch_all(reduce_scatter_kernel<Ty, OP, kVptReduce, kGroup>, p, work, s);
        case kOneshotTree:
            if (p.n <= 2) return launch_all(oneshot_tree_kernel<Ty, OP, 2, 8>, p, work, s);
            if (p.n <= 4) return launch_all(oneshot_tree_kernel<Ty, OP, 4, 4>, p, work, s);
            if (p.n <= 8) return launch_all(oneshot_tree_kernel<Ty, OP, 8, kVptReduce>, p, work, s);
            return launch_all(oneshot_tree_kernel<Ty, OP, kMaxRanks, kVptReduce>, p, work, s);
        case kAllGather: return launch_all(all_gather_kernel<Ty>, p, work, s);
        case kAllToAll: return launch_all(all_to_all_kernel<Ty>, p, work, s);
        case kChunkBroadcast: return launch_all(chunk_bcast_kernel<Ty>, p, work, s);
        }
        return cudaErrorInvalidValue;
    });
}

cudaError_t launch_step(int dtype, int op, const StepParams& p, cudaStream_t s)
{
    const uint64_t work = (uint64_t)p.nseg * p.tps;
    if (p.nin == 1) op = kSum;
    return with_type(dtype, op,
                     [&]<class Ty, int OP>() { return launch_all(step_kernel<Ty, OP>, p, work, s); });
}

}  // namespace rr
