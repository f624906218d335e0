// rr_bulk.cuh -- N-input folds whose tiles are staged in shared memory by
// the bulk async copy engine (cp.async.bulk) instead of per-thread 128-bit
// loads: one elected thread issues the N input copies of a tile behind an
// mbarrier, the CTA folds the tile in shared memory, and the same thread
// issues the bulk stores of the result.  Three orders and output patterns:
//
//   kBulkRing     the one-shot all-reduce: segment c = chunk c of every
//                 rank (clipped to the launch's element range), folded in
//                 ring order from rank c (optionally with the bf16 wire
//                 format), written to every rank or to rank c only (the
//                 two-shot's first shot)
//   kBulkScatter  the reduce-scatter: segment r = part r of every rank,
//                 folded in ring order from rank r, written to out[r] only
//   kBulkTree     the tree-order one-shot: the whole buffer, folded in the
//                 tree's pairwise order (an unpaired rank carried up), written
//                 to every rank
//
// The ring and tree modes run wherever every input and output address has
// the same 16-byte phase (a scalar head and tail per segment, whole vectors
// between), the scatter mode wherever every input has one phase (each output
// stored by bulk copies when it shares that phase, by the threads
// otherwise); ring and scatter for 2-64 ranks, tree for 2-8, 12 and 16
// (bulk_*_eligible).  The rank count is a compile-time constant for 2, 4, 8,
// 16, 32 and 64 ranks (tree: 2-8, 12 and 16) and a kernel argument (NS = 0)
// otherwise; with the copy engine doing the loads,
// a runtime count costs the fold no registers.  Every other call takes the
// per-thread-load kernels, with the same bits.  The fold itself uses the
// same apply / finish / wire steps as those kernels.
//
// Every mbarrier wait is bounded, and its outcome is the same in every thread
// of the CTA (bulk_tile_landed).  A tile whose wait runs out (no working
// device lets it) is skipped by the whole CTA -- nothing of it is stored --
// and counted in BulkParams::waits[0]; one thread then waits once more
// (bounded) for the tile's copies to land before the CTA leaves, and counts
// the tile in waits[1] if they were not seen to land (its shared memory may
// then still receive them after the CTA has left, so a nonzero waits[1]
// means the device is not usable).  rr_check_timeouts() takes both counts.
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "The five primitives", "Ring all-reduce and communication volume"
// and "alpha-beta model"; [P3] "Training gradient sync and collective
// communication" (geek-doc.cn), section 6 (the tree's pairwise order).
#pragma once

#include "rr_oneshot.cuh"

namespace rr {

enum BulkMode : int { kBulkRing = 0, kBulkScatter = 1, kBulkTree = 2 };

struct BulkParams {
    RankParams r;
    unsigned int* waits;  // device counters: [0] tiles whose wait ran out, [1] of those, tiles
                          // whose copies were not seen to land before the CTA left
    uint32_t hold;        // test hook (0 in use): 1 makes every barrier expect one arrival
                          // more, which is made only after the first wait has run out
    uint32_t spin;        // try_wait rounds before a wait gives up
    uint32_t tv;          // vectors per rank per tile (kernels whose rank count is not fixed)
};

// Bytes of input tiles per CTA (N tiles of a share each): 16 KB, 32 KB from
// kBulkWideRanks ranks on (so that a CTA keeps enough bytes in flight while
// it folds), and for a rank count given at run time kBulkManyBytes from 32
// ranks on.  Measured on 64 Mi fp32 per rank: 32 KB from 9 ranks instead of
// from 32 took 17-31 ranks from 0.83-0.97 to 1.00 of the copy peak; 40 KB
// took the run-time-count folds at 40-64 ranks up by 1-3 % and the
// compiled 32- and 64-rank ones down by 2 %.
#ifndef RR_BULK_WIDE_RANKS
#define RR_BULK_WIDE_RANKS 9
#endif
#ifndef RR_BULK_MANY_BYTES
#define RR_BULK_MANY_BYTES 40960
#endif
constexpr int kBulkWideRanks = RR_BULK_WIDE_RANKS;
constexpr uint32_t kBulkManyBytes = RR_BULK_MANY_BYTES;
static_assert(kBulkManyBytes + 64 <= 48 * 1024, "within the default dynamic shared memory of a CTA");

// Compiled rank counts.
template <int NS>
__host__ __device__ constexpr uint32_t bulk_smem()
{
    return NS >= kBulkWideRanks ? 32768u : 16384u;
}

// The parameter block of a launch: p, the counters' address (p.waits) and
// the wait bounds (rr_bulk.cu).
BulkParams bulk_params(const RankParams& p);

// Whether a call can take the aligned bulk kernels (scatter and tree modes):
// the wait counters are known (p.waits), 2..nmax ranks (powers of two only
// when pow2), 16-byte aligned buffers.  The callers add their own segment
// rules.
bool bulk_ranks_aligned(const RankParams& p, int nmax, bool pow2);

__device__ __forceinline__ uint32_t bulk_smem_addr(const void* ptr) { return (uint32_t)__cvta_generic_to_shared(ptr); }

__device__ __forceinline__ bool bulk_bar_wait(uint32_t bar, uint32_t parity, uint32_t spin)
{
    for (uint32_t i = 0; i < spin; ++i) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}

// Thread 0: set up a tile's barrier.  It completes once `1 + hold`
// arrivals have been made and the copies' bytes have landed.
__device__ __forceinline__ void bulk_bar_init(uint32_t bar, uint32_t hold)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(1u + hold) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Thread 0, once no thread waits on the barrier and no copy signals it.
__device__ __forceinline__ void bulk_bar_inval(uint32_t bar)
{
    asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Every thread of the CTA: wait (bounded) for the tile's copies.  Returns the
// same answer in every thread: true when every thread saw them land.  On
// false the CTA must skip the tile and leave; thread 0 has then counted the
// tile, made the arrival the test hook withheld, and waited (bounded) for the
// copies to land -- invalidating the barrier if they did, counting the tile
// in waits[1] if not -- so the CTA's shared memory is not left to a copy
// still in flight.
__device__ __forceinline__ bool bulk_tile_landed(uint32_t bar, unsigned int* waits, uint32_t hold, uint32_t spin)
{
    if (__syncthreads_and(bulk_bar_wait(bar, 0, spin))) return true;
    if (threadIdx.x == 0) {
        atomicAdd(&waits[0], 1u);
        if (hold) asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
        if (bulk_bar_wait(bar, 0, spin)) bulk_bar_inval(bar);
        else atomicAdd(&waits[1], 1u);
    }
    return false;
}

template <class Ty, int OP, int NS, int MODE, int WIRE>
__global__ void __launch_bounds__(kThreads) bulk_fold_kernel(const __grid_constant__ BulkParams bp)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;  // elements per 16-byte vector
    static_assert(NS == 0 || bulk_smem<NS>() / (NS > 0 ? NS : 1) >= 16, "a tile of at least one vector per rank");
    static_assert(MODE != kBulkTree || NS > 0, "the pairwise tree needs a fixed rank count");
    static_assert(MODE == kBulkRing || WIRE == 0, "the wire format is a ring-order one-shot");
    const RankParams& p = bp.r;
    const int n = NS > 0 ? NS : p.n;
    const uint32_t TV = NS > 0 ? bulk_smem<NS>() / (NS > 0 ? NS : 1) / 16 : bp.tv;  // vectors per rank per tile
    extern __shared__ __align__(128) uint4 sm[];                      // [n][TV]: slot j holds the fold's j-th input
    __shared__ __align__(8) uint64_t bar;

    const uint64_t s = blockIdx.x / p.tps, tile = blockIdx.x - s * p.tps;
    uint64_t lo, len;
    if constexpr (MODE == kBulkTree) {
        lo = 0;
        len = p.count;
    } else if constexpr (MODE == kBulkScatter) {
        lo = s * p.C;
        len = p.C;
    } else {  // chunk s, clipped to the launch's element range [p.lo, p.hi)
        const uint64_t c_lo = s * p.C;
        if (c_lo >= p.count) return;
        const uint64_t c_hi = p.C < p.count - c_lo ? c_lo + p.C : p.count;
        lo = c_lo > p.lo ? c_lo : p.lo;
        const uint64_t hi = c_hi < p.hi ? c_hi : p.hi;
        if (lo >= hi) return;
        len = hi - lo;
    }
    const int start = MODE == kBulkTree ? 0 : (int)s;
    auto in = [&](int j) {
        int r = start + j;
        if (r >= n) r -= n;
        return static_cast<const T*>(p.in[r]) + lo;
    };
    const bool one_out = MODE == kBulkScatter || (MODE == kBulkRing && p.owner_only);
    const int nout = one_out ? 1 : n;
    auto out = [&](int o) {
        if constexpr (MODE == kBulkScatter) return static_cast<T*>(p.out[s]);
        else return static_cast<T*>(p.out[one_out ? start : o]) + lo;
    };
    // Every rank's copy of the segment starts at the same 16-byte phase, so
    // the elements before the first 16-byte boundary (the head) and after the
    // last whole vector (the tail) are folded with plain loads by tile 0 (in
    // the tree's order in tree mode), and the bulk copies move the whole
    // vectors between.
    uint64_t head = (uint64_t)((L - phase_of(in(0), L)) & (L - 1));
    if (head > len) head = len;
    // a scatter output at another phase than the inputs is stored by the
    // threads, element by element, instead of by bulk stores
    bool bulk_out = true;
    if constexpr (MODE == kBulkScatter) bulk_out = phase_of(out(0), L) == phase_of(in(0), L);
    const uint64_t nv = (len - head) / L;  // whole vectors of the segment
    const uint64_t tail = len - head - nv * L;
    if (tile == 0 && (uint64_t)threadIdx.x < head + tail) {
        const uint64_t e = (uint64_t)threadIdx.x < head ? (uint64_t)threadIdx.x : head + nv * L + (threadIdx.x - head);
        if constexpr (MODE == kBulkTree) tree_fold_lanes<Ty, OP, 1, NS>(p, e, false);  // lo = 0
        else fold_one<Ty, OP, WIRE>(in, n, out, nout, e, p.divisor);
    }
    const uint64_t v0 = tile * TV;
    if (v0 >= nv) return;
    const uint32_t nvt = (uint32_t)(nv - v0 < TV ? nv - v0 : TV);  // vectors in this tile
    const uint32_t bytes = nvt * 16u;
    const uint64_t e0 = head + v0 * L;     // first element of the tile: 16-byte aligned in every copy

    const uint32_t b = bulk_smem_addr(&bar);
    if (threadIdx.x == 0) bulk_bar_init(b, bp.hold);
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                     ::"r"(b), "r"(bytes * (uint32_t)n) : "memory");
#pragma unroll
        for (int j = 0; j < (NS > 0 ? NS : n); ++j)
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                ::"r"(bulk_smem_addr(sm + j * TV)), "l"(in(j) + e0), "r"(bytes), "r"(b)
                : "memory");
    }
    if (!bulk_tile_landed(b, bp.waits, bp.hold, bp.spin)) return;  // the whole CTA skips the tile
    for (uint32_t v = threadIdx.x; v < nvt; v += kThreads) {
        Acc a[L];
        if constexpr (MODE == kBulkTree) {
            // pairwise order with fp32 partials: slot j joins a stack whose
            // level b holds a finished block of 2^b ranks (no rounding between
            // levels).  After the last slot the stack holds one block per set
            // bit of N; the tree carries an unpaired block up until a level
            // pairs it, so the blocks combine from the lowest level upwards,
            // each higher block on the left (one block of all ranks when N is
            // a power of two).
            constexpr int LV = NS <= 2 ? 2 : NS <= 4 ? 3 : NS <= 8 ? 4 : NS <= 16 ? 5 : NS <= 32 ? 6 : 7;
            Acc stack[LV][L];
#pragma unroll
            for (int j = 0; j < NS; ++j) {
                Ty::unpack(sm[j * TV + v], a);
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
                if (!((NS >> bb) & 1)) continue;
#pragma unroll
                for (int l = 0; l < L; ++l) a[l] = have ? apply<OP>(stack[bb][l], a[l]) : stack[bb][l];
                have = true;
            }
        } else {
            Ty::unpack(sm[v], a);
#pragma unroll 4
            for (int j = 1; j < (NS > 0 ? NS : n); ++j) {
                Acc x[L];
                Ty::unpack(sm[j * TV + v], x);
#pragma unroll
                for (int l = 0; l < L; ++l) a[l] = apply<OP>(wire_in<WIRE>(a[l]), x[l]);
            }
        }
#pragma unroll
        for (int l = 0; l < L; ++l) a[l] = wire_out<WIRE>(finish_n<OP, NS>(a[l], p.divisor));
        sm[v] = Ty::pack(a);  // into slot 0, which this thread has read
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the generic writes, before the bulk reads
    __syncthreads();
    if (!bulk_out) {
        for (uint32_t v = threadIdx.x; v < nvt; v += kThreads) st_lanes(out(0) + e0 + (uint64_t)v * L, sm[v]);
        if (threadIdx.x == 0) bulk_bar_inval(b);
        return;
    }
    if (threadIdx.x == 0) {
        for (int o = 0; o < nout; ++o)
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                         ::"l"(out(o) + e0), "r"(bulk_smem_addr(sm)), "r"(bytes)
                         : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // slot 0 read before the CTA leaves
        bulk_bar_inval(b);
    }
}

// Vectors per rank per tile when the rank count is not fixed at compile
// time: the rank's share of the tile bytes, whole vectors.
inline uint32_t bulk_tile_vectors(int n)
{
    const uint32_t bytes = n >= 32 ? kBulkManyBytes : n >= kBulkWideRanks ? 32768u : 16384u;
    return bytes / (uint32_t)n / 16u;
}

// The same for a launch that may take a compiled rank count (the ring mode
// compiles 32 and 64 ranks; below 32 the two tilings agree).
inline uint32_t bulk_launch_tile_vectors(int n)
{
    if (n == 32) return bulk_smem<32>() / 32u / 16u;
    if (n == 64) return bulk_smem<64>() / 64u / 16u;
    return bulk_tile_vectors(n);
}

// One CTA per (segment, tile): nseg segments of at most seg_elems elements
// each.  NS = 0 runs the rank count p.n.
template <class Ty, int OP, int NS, int MODE, int WIRE>
cudaError_t launch_bulk_fold(const RankParams& p, uint64_t seg_elems, cudaStream_t s)
{
    BulkParams bp = bulk_params(p);
    if (!bp.waits) return cudaErrorInvalidValue;  // never reached: eligibility requires the counters
    const uint32_t tv = NS > 0 ? bulk_smem<NS>() / (NS > 0 ? NS : 1) / 16 : bulk_tile_vectors(p.n);
    const uint64_t te = (uint64_t)tv * Ty::L;  // elements per tile
    bp.tv = tv;
    bp.r.tps = seg_elems ? (seg_elems + te - 1) / te : 1;
    const uint64_t work = bp.r.nseg * bp.r.tps;
    if (work == 0) return cudaSuccess;
    if (work > kMaxGrid) return cudaErrorInvalidValue;  // never reached: the eligibility checks cap it
    const uint32_t smem = tv * 16u * (uint32_t)p.n;
    bulk_fold_kernel<Ty, OP, NS, MODE, WIRE><<<(unsigned)work, kThreads, smem, s>>>(bp);
    return cudaGetLastError();
}

}  // namespace rr
