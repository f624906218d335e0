// rr_bulk.cu -- the one-shot all-reduce in ring order with its tiles staged
// in shared memory by the bulk async copy engine (cp.async.bulk) instead of
// per-thread 128-bit loads: one elected thread issues the N input copies of
// a tile behind an mbarrier, the CTA folds the tile in shared memory in ring
// order, and the same thread issues the N bulk stores of the result.
//
// It runs where the tiles are whole 16-byte vectors at 16-byte aligned
// addresses: every buffer 16-byte aligned, the chunk size a multiple of 16
// bytes, a plain in-place call, and a rank count fixed at compile time (2, 4,
// 8, 16, 32, 64).  The few elements past a ragged chunk's last whole vector are
// folded with plain loads.  Same bits as oneshot_ring_kernel.  Measured on
// 8 x 256 MiB fp32: 1.04-1.05 of the copy peak against 1.03 for the
// per-thread loads.
//
// Every mbarrier wait is bounded.  A wait that runs out (no working device
// lets it) skips its tile, counts itself in g_bulk_timeouts, waits once more
// (bounded) for its own copies in flight and returns; rr_check_timeouts()
// reads and clears the count.
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "Ring all-reduce and communication volume" and "alpha-beta model".
#include <cstdlib>
#include <cstring>

#include "rr_oneshot.cuh"

namespace rr {

namespace {

__device__ unsigned int g_bulk_timeouts = 0;

// Bytes of input tiles per CTA (N tiles of bulk_smem<N>() / N): 16 KB, 32 KB
// from 32 ranks on so that each rank's tile stays at least 512 bytes.
template <int NS>
__host__ __device__ constexpr uint32_t bulk_smem()
{
    return NS >= 32 ? 32768u : 16384u;
}

// Test hook, read once per process: RR_DEBUG_BULK_TIMEOUT=1 makes every
// barrier expect 16 bytes more than its copies bring and bounds each wait at
// 2^16 rounds, so that every wait runs out (the copies themselves complete,
// long before the second wait ends).
struct BulkDebug {
    uint32_t extra_tx = 0;
    uint32_t spin = 1u << 22;  // try_wait rounds, each of which may suspend the thread briefly
    BulkDebug()
    {
        const char* v = std::getenv("RR_DEBUG_BULK_TIMEOUT");
        if (v && std::strcmp(v, "1") == 0) {
            extra_tx = 16;
            spin = 1u << 16;
        }
    }
};

const BulkDebug& bulk_debug()
{
    static const BulkDebug d;
    return d;
}

struct BulkParams {
    RankParams r;
    uint32_t extra_tx;
    uint32_t spin;
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, uint32_t spin)
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

template <class Ty, int OP, int NS>
__global__ void __launch_bounds__(kThreads) oneshot_bulk_kernel(const __grid_constant__ BulkParams bp)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;                       // elements per 16-byte vector
    constexpr uint32_t TB = bulk_smem<NS>() / NS;  // bytes per rank per tile
    constexpr uint32_t TV = TB / 16;               // vectors per tile
    static_assert(TB % 16 == 0 && TV >= 1, "tile of whole vectors");
    const RankParams& p = bp.r;
    extern __shared__ __align__(128) uint4 sm[];   // [NS][TV]: slot j holds rank (c + j) mod N
    __shared__ __align__(8) uint64_t bar;

    const uint64_t c = blockIdx.x / p.tps, tile = blockIdx.x - c * p.tps;
    const uint64_t lo = c * p.C;
    if (lo >= p.count) return;
    const uint64_t len = p.C < p.count - lo ? p.C : p.count - lo;
    const uint64_t nv = len / L;                   // whole vectors of the chunk
    const int start = (int)c;
    auto in = [&](int j) {
        int r = start + j;
        if (r >= NS) r -= NS;
        return static_cast<const T*>(p.in[r]) + lo;
    };
    auto out = [&](int o) { return static_cast<T*>(p.out[o]) + lo; };
    if (tile == 0 && (uint64_t)threadIdx.x < len - nv * L)  // the elements past the last whole vector
        fold_one<Ty, OP, 0>(in, NS, out, NS, nv * L + threadIdx.x, p.divisor);
    const uint64_t v0 = tile * TV;
    if (v0 >= nv) return;
    const uint32_t nvt = (uint32_t)(nv - v0 < TV ? nv - v0 : TV);  // vectors in this tile
    const uint32_t bytes = nvt * 16u;
    const uint64_t e0 = v0 * L;                    // first element of the tile in the chunk

    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                     ::"r"(b), "r"(bytes * NS + bp.extra_tx) : "memory");
#pragma unroll
        for (int j = 0; j < NS; ++j)
            asm volatile(
                "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                ::"r"(smem_addr(sm + j * TV)), "l"(in(j) + e0), "r"(bytes), "r"(b)
                : "memory");
    }
    if (!bar_wait(b, 0, bp.spin)) {
        if (threadIdx.x == 0) atomicAdd(&g_bulk_timeouts, 1u);
        bar_wait(b, 0, bp.spin);  // once more for the copies in flight, then leave the tile
        return;
    }
    // fold every vector of the tile in ring order, in place in slot 0
    for (uint32_t v = threadIdx.x; v < nvt; v += kThreads) {
        Acc a[L];
        Ty::unpack(sm[v], a);
#pragma unroll
        for (int j = 1; j < NS; ++j) {
            Acc x[L];
            Ty::unpack(sm[j * TV + v], x);
#pragma unroll
            for (int l = 0; l < L; ++l) a[l] = apply<OP>(a[l], x[l]);
        }
#pragma unroll
        for (int l = 0; l < L; ++l) a[l] = finish_n<OP, NS>(a[l], p.divisor);
        sm[v] = Ty::pack(a);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the generic writes, before the bulk reads
    __syncthreads();
    if (threadIdx.x == 0) {
#pragma unroll
        for (int o = 0; o < NS; ++o)
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                         ::"l"(out(o) + e0), "r"(smem_addr(sm)), "r"(bytes)
                         : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // slot 0 read before the CTA leaves
    }
}

template <class Ty, int OP, int NS>
cudaError_t launch_bulk(const RankParams& p, cudaStream_t s)
{
    constexpr uint64_t TE = (uint64_t)(bulk_smem<NS>() / NS / 16) * Ty::L;  // elements per tile
    BulkParams bp{};
    bp.r = p;
    bp.r.tps = (p.C + TE - 1) / TE;
    bp.extra_tx = bulk_debug().extra_tx;
    bp.spin = bulk_debug().spin;
    const uint64_t work = bp.r.nseg * bp.r.tps;
    if (work == 0) return cudaSuccess;
    if (work > kMaxGrid) return cudaErrorInvalidValue;  // never reached: bulk_eligible caps the grid
    oneshot_bulk_kernel<Ty, OP, NS><<<(unsigned)work, kThreads, bulk_smem<NS>(), s>>>(bp);
    return cudaGetLastError();
}

}  // namespace

bool bulk_eligible(const RankParams& p, int esize)
{
    if (p.n != 2 && p.n != 4 && p.n != 8 && p.n != 16 && p.n != 32 && p.n != 64) return false;
    if (p.owner_only || p.lo != 0 || p.hi < p.count || p.nseg != (uint64_t)p.n) return false;
    if ((p.C * (uint64_t)esize) % 16 != 0) return false;
    for (int r = 0; r < p.n; ++r)
        if ((uintptr_t)p.in[r] % 16 != 0 || (uintptr_t)p.out[r] % 16 != 0) return false;
    const uint64_t tb = (p.n >= 32 ? 32768u : 16384u) / (uint64_t)p.n;  // bulk_smem<N>() / N
    const uint64_t tiles = (p.C * (uint64_t)esize + tb - 1) / tb;
    return tiles * (uint64_t)p.n <= kMaxGrid;
}

template <class Ty, int OP>
cudaError_t launch_oneshot_bulk(const RankParams& p, cudaStream_t s)
{
    switch (p.n) {
    case 2: return launch_bulk<Ty, OP, 2>(p, s);
    case 4: return launch_bulk<Ty, OP, 4>(p, s);
    case 8: return launch_bulk<Ty, OP, 8>(p, s);
    case 16: return launch_bulk<Ty, OP, 16>(p, s);
    case 32: return launch_bulk<Ty, OP, 32>(p, s);
    case 64: return launch_bulk<Ty, OP, 64>(p, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t take_bulk_timeouts(unsigned int* count)
{
    cudaError_t e = cudaMemcpyFromSymbol(count, g_bulk_timeouts, sizeof(unsigned int));
    if (e != cudaSuccess) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_bulk_timeouts, &zero, sizeof(unsigned int));
}

#define RR_INSTANTIATE(TY, OP) template cudaError_t launch_oneshot_bulk<TY, OP>(const RankParams&, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_INSTANTIATE)
#undef RR_INSTANTIATE

}  // namespace rr
