// rr_bulk.cuh -- N-input folds whose tiles are staged in shared memory by
// the bulk async copy engine (cp.async.bulk) instead of per-thread 128-bit
// loads: one elected thread issues the N input copies of a tile behind an
// mbarrier, the CTA folds the tile in shared memory, and the same thread
// issues the bulk stores of the result.  Three orders and output patterns:
//
//   kBulkRing     the one-shot all-reduce: segment c = chunk c of every
//                 rank, folded in ring order from rank c (optionally with the
//                 bf16 wire format), written to every rank
//   kBulkScatter  the reduce-scatter: segment r = part r of every rank,
//                 folded in ring order from rank r, written to out[r] only
//   kBulkTree     the tree-order one-shot: the whole buffer, folded in the
//                 tree's pairwise order (N a power of two), written to every
//                 rank
//
// They run where the tiles are whole 16-byte vectors at 16-byte aligned
// addresses and the rank count is fixed at compile time (bulk_*_eligible);
// every other call takes the per-thread-load kernels, with the same bits.
// The fold itself uses the same apply / finish / wire steps as those kernels.
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
};

// Bytes of input tiles per CTA (N tiles of bulk_smem<N>() / N): 16 KB, 32 KB
// from 32 ranks on so that each rank's tile stays at least 512 bytes.
template <int NS>
__host__ __device__ constexpr uint32_t bulk_smem()
{
    return NS >= 32 ? 32768u : 16384u;
}

// The parameter block of a launch: p, the counters' address (p.waits) and
// the wait bounds (rr_bulk.cu).
BulkParams bulk_params(const RankParams& p);

// Whether a call can take the bulk kernels: the wait counters are known
// (p.waits), a rank count of 2, 4, 8, 16, 32 or 64 (up to nmax), 16-byte
// aligned buffers.  The callers add their own segment rules.
bool bulk_ranks_aligned(const RankParams& p, int nmax);

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
    constexpr int L = Ty::L;                       // elements per 16-byte vector
    constexpr uint32_t TB = bulk_smem<NS>() / NS;  // bytes per rank per tile
    constexpr uint32_t TV = TB / 16;               // vectors per tile
    constexpr int NOUT = MODE == kBulkScatter ? 1 : NS;
    static_assert(TB % 16 == 0 && TV >= 1, "tile of whole vectors");
    static_assert(MODE != kBulkTree || (NS & (NS - 1)) == 0, "the pairwise tree needs a power of two");
    const RankParams& p = bp.r;
    extern __shared__ __align__(128) uint4 sm[];   // [NS][TV]: slot j holds the fold's j-th input
    __shared__ __align__(8) uint64_t bar;

    const uint64_t s = blockIdx.x / p.tps, tile = blockIdx.x - s * p.tps;
    uint64_t lo, len;
    if constexpr (MODE == kBulkTree) {
        lo = 0;
        len = p.count;
    } else {
        lo = s * p.C;
        if (lo >= p.count) return;
        len = p.C < p.count - lo ? p.C : p.count - lo;
    }
    const int start = MODE == kBulkTree ? 0 : (int)s;
    auto in = [&](int j) {
        int r = start + j;
        if (r >= NS) r -= NS;
        return static_cast<const T*>(p.in[r]) + lo;
    };
    auto out = [&](int o) {
        if constexpr (MODE == kBulkScatter) return static_cast<T*>(p.out[s]);
        else return static_cast<T*>(p.out[o]) + lo;
    };
    const uint64_t nv = len / L;                   // whole vectors of the segment
    if constexpr (MODE == kBulkRing) {             // a ragged last chunk: its last elements
        if (tile == 0 && (uint64_t)threadIdx.x < len - nv * L)
            fold_one<Ty, OP, WIRE>(in, NS, out, NOUT, nv * L + threadIdx.x, p.divisor);
    }
    const uint64_t v0 = tile * TV;
    if (v0 >= nv) return;
    const uint32_t nvt = (uint32_t)(nv - v0 < TV ? nv - v0 : TV);  // vectors in this tile
    const uint32_t bytes = nvt * 16u;
    const uint64_t e0 = v0 * L;                    // first element of the tile in the segment

    const uint32_t b = bulk_smem_addr(&bar);
    if (threadIdx.x == 0) bulk_bar_init(b, bp.hold);
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                     ::"r"(b), "r"(bytes * NS) : "memory");
#pragma unroll
        for (int j = 0; j < NS; ++j)
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
            // level b holds a finished block of 2^b ranks (no rounding between levels)
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
#pragma unroll
            for (int l = 0; l < L; ++l) a[l] = stack[LV - 1][l];  // N = 2^(LV-1): one block of all ranks
        } else {
            Ty::unpack(sm[v], a);
#pragma unroll
            for (int j = 1; j < NS; ++j) {
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
    if (threadIdx.x == 0) {
#pragma unroll
        for (int o = 0; o < NOUT; ++o)
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                         ::"l"(out(o) + e0), "r"(bulk_smem_addr(sm)), "r"(bytes)
                         : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // slot 0 read before the CTA leaves
        bulk_bar_inval(b);
    }
}

// One CTA per (segment, tile): nseg segments of seg_elems elements each.
template <class Ty, int OP, int NS, int MODE, int WIRE>
cudaError_t launch_bulk_fold(const RankParams& p, uint64_t seg_elems, cudaStream_t s)
{
    constexpr uint64_t TE = (uint64_t)(bulk_smem<NS>() / NS / 16) * Ty::L;  // elements per tile
    BulkParams bp = bulk_params(p);
    if (!bp.waits) return cudaErrorInvalidValue;  // never reached: eligibility requires the counters
    bp.r.tps = (seg_elems + TE - 1) / TE;
    const uint64_t work = bp.r.nseg * bp.r.tps;
    if (work == 0) return cudaSuccess;
    if (work > kMaxGrid) return cudaErrorInvalidValue;  // never reached: the eligibility checks cap it
    bulk_fold_kernel<Ty, OP, NS, MODE, WIRE><<<(unsigned)work, kThreads, bulk_smem<NS>(), s>>>(bp);
    return cudaGetLastError();
}

}  // namespace rr
