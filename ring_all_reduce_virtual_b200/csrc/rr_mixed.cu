// rr_mixed.cu -- the one-shot all-reduce (ring order, its two-shot first
// shot and bf16-wire form, and tree order) and the reduce-scatter over rank
// buffers whose addresses differ modulo 16 bytes (views at unequal offsets):
// no 16-byte vector of one rank lines up with the same elements of another.
//
// Each CTA takes one tile of one segment (a chunk, a part, or in tree order
// the whole buffer).  Every rank's elements of the tile are copied by
// cp.async into a shared-memory slot of its own, as the aligned 16-byte
// vectors that cover them (the slot remembers where the first element
// sits); the fold takes the tile's m-th vector of elements from every slot --
// shifted out of the two slot vectors it straddles -- in ring order and
// writes the rounded result into a result slot, element 0 first; each output
// gets whole aligned 16-byte stores, every vector shifted out of two result
// vectors to the output's phase, plus scalar stores for the elements before
// its first 16-byte boundary and after its last whole vector.  Same bits as
// the aligned kernels (the fold, finish and rounding steps of rr_device.cuh).
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "The five primitives", "Ring all-reduce and communication volume"
// and "alpha-beta model" (one-shot: every rank reads every peer's buffer
// directly); [P3] "Training gradient sync and collective communication"
// (geek-doc.cn), section 6 (tree order); [P1] "How all-reduce keeps every card
// identical" (mhpq.cn), section 7.3 (low-precision gradients on the wire).
#include "rr_bulk.cuh"

namespace rr {

namespace {

// Vectors of input per rank per tile: as for the bulk-copy folds (a rank's
// share of 16 KB, 32 KB from 9 ranks on, 40 KB from 32), so that the slots and
// the result stay within the 48 KB a CTA gets by default.
uint32_t mixed_tile_vectors(int n)
{
    return bulk_tile_vectors(n);
}

struct MixedParams {
    RankParams r;
    uint32_t tv;  // vectors per rank per tile; every slot holds tv + 1
    uint32_t pad_;
};

// MODE kMixedRing: segment c = chunk c of every rank, folded from rank c,
// written to every rank (or to rank c only: the two-shot's first shot);
// kMixedScatter: segment r = part r (offset r*C) of every rank, folded from
// rank r, written to out[r] (the reduce-scatter); kMixedTree: the whole
// buffer as one segment, folded in the tree's pairwise order (up to 16
// ranks), written to every rank.  WIRE: the bf16 wire format of the
// ring-order one-shot (rr_device.cuh).
enum MixedMode : int { kMixedRing = 0, kMixedScatter = 1, kMixedTree = 2 };

// TMAX: the most ranks a tree-mode instance folds (8 or 16; its stack holds
// one level per power of two).
template <class Ty, int OP, int MODE, int WIRE, int TMAX = 16>
__global__ void __launch_bounds__(kThreads) oneshot_mixed_kernel(const __grid_constant__ MixedParams mp)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;
    const RankParams& p = mp.r;
    const int n = p.n;
    const uint32_t TV = mp.tv, SV = TV + 1;
    const uint64_t TE = (uint64_t)TV * L;  // elements per tile
    extern __shared__ __align__(16) uint4 sm[];  // [n][SV] rank slots, then [SV] result
    __shared__ uint32_t shift[kMaxRanks];        // slot j's first element of the tile

    const uint64_t c = blockIdx.x / p.tps, tile = blockIdx.x - c * p.tps;
    uint64_t lo, hi;
    if constexpr (MODE == kMixedScatter) {
        lo = c * p.C;
        hi = lo + p.C;
    } else if constexpr (MODE == kMixedTree) {
        lo = 0;
        hi = p.count;
    } else {  // chunk c clipped to this launch's element range
        const uint64_t c_lo = c * p.C;
        if (c_lo >= p.count) return;
        const uint64_t c_hi = p.C < p.count - c_lo ? c_lo + p.C : p.count;
        lo = c_lo > p.lo ? c_lo : p.lo;
        hi = c_hi < p.hi ? c_hi : p.hi;
    }
    const uint64_t start = lo + tile * TE;
    if (lo >= hi || start >= hi) return;
    const uint32_t te = (uint32_t)(hi - start < TE ? hi - start : TE);  // elements of this tile
    const int first = (int)c;
    auto in = [&](int j) {
        int r = first + j;
        if (r >= n) r -= n;
        return static_cast<const T*>(p.in[r]) + start;
    };
    const int nout = MODE == kMixedScatter || (MODE == kMixedRing && p.owner_only) ? 1 : n;
    auto out = [&](int o) {
        if constexpr (MODE == kMixedScatter) return static_cast<T*>(p.out[first]) + (start - lo);
        else if constexpr (MODE == kMixedTree) return static_cast<T*>(p.out[o]) + start;
        else return static_cast<T*>(p.out[p.owner_only ? first : o]) + start;
    };

    // 1. stage: slot j holds rank (c + j) mod N, from the aligned vector at or
    // below the tile's first element up to the one holding its last element;
    // every vector copied holds an element of the tile, so no copy leaves the
    // 16-byte blocks of the rank's buffer
    if (threadIdx.x < (unsigned)n) shift[threadIdx.x] = (uint32_t)(((uintptr_t)in(threadIdx.x) & 15u) / sizeof(T));
    for (uint32_t q = threadIdx.x; q < (uint32_t)n * SV; q += kThreads) {
        const uint32_t j = q / SV, v = q - j * SV;
        const T* b = in((int)j);
        const uint32_t sh = (uint32_t)(((uintptr_t)b & 15u) / sizeof(T));
        if (v * L < sh + te)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(&sm[q])),
                         "l"(reinterpret_cast<const uint4*>((uintptr_t)b & ~(uintptr_t)15u) + v)
                         : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();

    // 2. fold the tile's m-th vector of elements in ring order into the result
    // slot (lanes past the tile's end are folded from whatever the slots hold
    // there and never stored)
    uint4* resv = sm + (uint32_t)n * SV;
    const T* res = reinterpret_cast<const T*>(resv);
    const uint32_t nvt = (te + L - 1) / L;
    auto slot_vec = [&](int j, uint32_t m) {
        const uint4* v = sm + (uint32_t)j * SV + m;
        const uint32_t sh = shift[j];
        return sh ? shift_window(v[0], v[1], (int)(sh * sizeof(T))) : v[0];
    };
    for (uint32_t m = threadIdx.x; m < nvt; m += kThreads) {
        Acc a[L];
        if constexpr (MODE == kMixedTree) {
            // the tree's pairwise order with fp32 partials: slot j joins a
            // stack whose level b holds a finished block of 2^b ranks; after
            // the last slot the blocks of the set bits of N combine from the
            // lowest level up, each higher (earlier) block on the left
            constexpr int LV = TMAX <= 8 ? 4 : 5;  // log2(TMAX) + 1 levels
            Acc stack[LV][L];
#pragma unroll
            for (int j = 0; j < TMAX; ++j) {
                if (j >= n) break;
                Ty::unpack(slot_vec(j, m), a);
                int lvl = 0;
#pragma unroll
                for (int bb = 0; bb < LV - 1; ++bb) {
                    if (((j >> bb) & 1) && lvl == bb) {
#pragma unroll
                        for (int l = 0; l < L; ++l) a[l] = apply<OP>(stack[bb][l], a[l]);
                        lvl = bb + 1;
                    }
                }
#pragma unroll
                for (int bb = 0; bb < LV; ++bb)
                    if (bb == lvl)
#pragma unroll
                        for (int l = 0; l < L; ++l) stack[bb][l] = a[l];
            }
            bool have = false;
#pragma unroll
            for (int bb = 0; bb < LV; ++bb) {
                if (!((n >> bb) & 1)) continue;
#pragma unroll
                for (int l = 0; l < L; ++l) a[l] = have ? apply<OP>(stack[bb][l], a[l]) : stack[bb][l];
                have = true;
            }
        } else {
            Ty::unpack(slot_vec(0, m), a);
            for (int j = 1; j < n; ++j) {
                Acc x[L];
                Ty::unpack(slot_vec(j, m), x);
#pragma unroll
                for (int l = 0; l < L; ++l) a[l] = apply<OP>(wire_in<WIRE>(a[l]), x[l]);
            }
        }
#pragma unroll
        for (int l = 0; l < L; ++l) a[l] = wire_out<WIRE>(finish<OP>(a[l], p.divisor));
        resv[m] = Ty::pack(a);
    }
    __syncthreads();

    // 3. every output: whole aligned vectors shifted out of the result (item
    // q = vector m of output o, all outputs' vectors spread over the CTA), and
    // scalars before the first 16-byte boundary and after the last whole vector.
    // Measured at 2 / 4 / 8 / 16 ranks x 256 MiB fp32: this walk 1.00 / 0.93 /
    // 0.89 / 0.955 of the copy peak; the same items found by a division per
    // item 0.82 / 0.80 / 0.78 / 0.96; one output after the other 1.01 / 0.96 /
    // 0.86 / 0.93.  Thread t takes items t, t + kThreads, ... of the (output,
    // vector) sequence, stepping through it without a division.
    {
        int o = 0;
        uint32_t m = threadIdx.x;
        while (o < nout && m >= nvt) m -= nvt, ++o;
        while (o < nout) {
            T* ob = out(o);
            uint32_t h = (uint32_t)((L - phase_of(ob, L)) & (L - 1));
            if (h > te) h = te;
            const uint32_t nv = (te - h) / L;
            for (; m < nvt; m += kThreads) {
                if (m >= nv) continue;  // past the output's last whole vector
                const uint4 v = h ? shift_window(resv[m], resv[m + 1], (int)(h * sizeof(T))) : resv[m];
                stv(ob + h + (uint64_t)m * L, v);
            }
            while (o < nout && m >= nvt) m -= nvt, ++o;
        }
    }
    for (uint32_t q = threadIdx.x; q < (uint32_t)nout * 2u * L; q += kThreads) {
        const uint32_t o = q / (2u * L), k = q - o * (2u * L);
        T* ob = out((int)o);
        uint32_t h = (uint32_t)((L - phase_of(ob, L)) & (L - 1));
        if (h > te) h = te;
        const uint32_t nv = (te - h) / L, tail = te - h - nv * L;
        if (k < h + tail) {
            const uint32_t e = k < h ? k : h + nv * L + (k - h);
            ob[e] = res[e];
        }
    }
}

}  // namespace

bool mixed_eligible(const RankParams& p, int esize)
{
    // any 2-64 ranks (measured against one element per access, fp32 / bf16
    // of the copy peak: 24 ranks 0.81 / 0.69 against 0.45 / 0.24, 64 ranks
    // 0.61 / 0.51 against 0.53-0.62 / 0.30)
    if (p.n < 2 || p.n > kMaxRanks || p.nseg != (uint64_t)p.n || p.lo >= p.count) return false;
    for (int r = 0; r < p.n; ++r)  // element boundaries (the API checks them too)
        if ((uintptr_t)p.in[r] % (uintptr_t)esize || (uintptr_t)p.out[r] % (uintptr_t)esize) return false;
    const uint64_t hi = p.hi < p.count ? p.hi : p.count;
    const uint64_t seg = hi - p.lo < p.C ? hi - p.lo : p.C;
    const uint64_t te = (uint64_t)mixed_tile_vectors(p.n) * (16u / (uint64_t)esize);
    return (seg + te - 1) / te * (uint64_t)p.n <= kMaxGrid;
}

bool mixed_tree_eligible(const RankParams& p, int esize)
{
    if (p.n < 2 || p.n > 16 || p.nseg != 1) return false;
    for (int r = 0; r < p.n; ++r)
        if ((uintptr_t)p.in[r] % (uintptr_t)esize || (uintptr_t)p.out[r] % (uintptr_t)esize) return false;
    const uint64_t te = (uint64_t)mixed_tile_vectors(p.n) * (16u / (uint64_t)esize);
    return (p.count + te - 1) / te <= kMaxGrid;
}

namespace {

// One CTA per (segment, tile); a segment is a chunk clipped to the launch's
// element range (ring mode), a part (scatter mode) or the whole buffer (tree
// mode).
template <class Ty, int OP, int MODE, int WIRE, int TMAX = 16>
cudaError_t launch_mixed(const RankParams& p, cudaStream_t s)
{
    MixedParams mp{};
    mp.r = p;
    mp.tv = mixed_tile_vectors(p.n);
    const uint64_t te = (uint64_t)mp.tv * Ty::L;
    uint64_t seg = MODE == kMixedTree ? p.count : p.C;
    if constexpr (MODE == kMixedRing) {
        const uint64_t hi = p.hi < p.count ? p.hi : p.count;
        seg = hi - p.lo < p.C ? hi - p.lo : p.C;
    }
    mp.r.tps = seg ? (seg + te - 1) / te : 1;
    const uint64_t work = p.nseg * mp.r.tps;
    if (work == 0) return cudaSuccess;
    if (work > kMaxGrid) return cudaErrorInvalidValue;  // never reached: mixed_eligible caps it
    const uint32_t smem = ((uint32_t)p.n + 1u) * (mp.tv + 1u) * 16u;
    oneshot_mixed_kernel<Ty, OP, MODE, WIRE, TMAX><<<(unsigned)work, kThreads, smem, s>>>(mp);
    return cudaGetLastError();
}

}  // namespace

template <class Ty, int OP>
cudaError_t launch_oneshot_mixed(const RankParams& p, cudaStream_t s)
{
    return launch_mixed<Ty, OP, kMixedRing, 0>(p, s);
}

template <class Ty, int OP>
cudaError_t launch_scatter_mixed(const RankParams& p, cudaStream_t s)
{
    return launch_mixed<Ty, OP, kMixedScatter, 0>(p, s);
}

template <class Ty, int OP>
cudaError_t launch_tree_mixed(const RankParams& p, cudaStream_t s)
{
    // a stack of 4 levels up to 8 ranks: 48 registers instead of 64 (fp32)
    return p.n <= 8 ? launch_mixed<Ty, OP, kMixedTree, 0, 8>(p, s) : launch_mixed<Ty, OP, kMixedTree, 0, 16>(p, s);
}

cudaError_t launch_oneshot_wire_mixed(int op, const RankParams& p, cudaStream_t s)
{
    return op == kAvg ? launch_mixed<F32T, kAvg, kMixedRing, 1>(p, s) : launch_mixed<F32T, kSum, kMixedRing, 1>(p, s);
}

#define RR_INSTANTIATE(TY, OP)                                                                   \
    template cudaError_t launch_oneshot_mixed<TY, OP>(const RankParams&, cudaStream_t);           \
    template cudaError_t launch_scatter_mixed<TY, OP>(const RankParams&, cudaStream_t);            \
    template cudaError_t launch_tree_mixed<TY, OP>(const RankParams&, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_INSTANTIATE)
#undef RR_INSTANTIATE

}  // namespace rr
