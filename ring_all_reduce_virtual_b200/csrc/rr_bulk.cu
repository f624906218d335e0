// rr_bulk.cu -- the bulk-copy one-shot all-reduce in ring order (and its
// bf16-wire form), the timeout counter of every bulk kernel, and the
// eligibility checks.  The kernel template is in rr_bulk.cuh.
//
// Measured on 8 x 256 MiB fp32: 1.047 of the copy peak against 1.033 for the
// per-thread-load one-shot (moving the loads to the copy engine leaves a
// thread 30 registers instead of 80, so 8 CTAs per SM keep their copies in
// flight instead of 3).
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "Ring all-reduce and communication volume" and "alpha-beta model".
#include <cstdlib>
#include <cstring>
#include <atomic>

#include "rr_bulk.cuh"

namespace rr {

namespace {

// [0] tiles whose bounded wait ran out, [1] of those, tiles whose copies
// were not seen to land; one pair per device (each device holds its own
// copy of the module's variables).
__device__ unsigned int g_bulk_waits[2] = {0u, 0u};
__device__ unsigned int g_bulk_taken[2] = {0u, 0u};

__global__ void take_waits_kernel()
{
    g_bulk_taken[0] = atomicExch(&g_bulk_waits[0], 0u);
    g_bulk_taken[1] = atomicExch(&g_bulk_waits[1], 0u);
}

// Test hook, read once per process: RR_DEBUG_BULK_TIMEOUT=1 makes every
// barrier expect one arrival more than the copying thread makes, and bounds
// each wait at 2^16 rounds, so that every first wait runs out; the missing
// arrival is then made, and the second wait ends when the tile's copies have
// landed -- the path a real timeout takes.
struct BulkDebug {
    uint32_t hold = 0;
    uint32_t spin = 1u << 22;  // try_wait rounds, each of which may suspend the thread briefly
    BulkDebug()
    {
        const char* v = std::getenv("RR_DEBUG_BULK_TIMEOUT");
        if (v && std::strcmp(v, "1") == 0) {
            hold = 1;
            spin = 1u << 16;
        }
    }
};

const BulkDebug& bulk_debug()
{
    static const BulkDebug d;
    return d;
}

template <class Ty, int OP, int WIRE>
cudaError_t launch_ring(const RankParams& p, cudaStream_t s)
{
    uint64_t seg = p.C;  // the longest segment: a chunk, or the launch's element range
    const uint64_t hi = p.hi < p.count ? p.hi : p.count;
    if (hi - p.lo < seg) seg = hi - p.lo;
    switch (p.n) {
    case 2: return launch_bulk_fold<Ty, OP, 2, kBulkRing, WIRE>(p, seg, s);
    case 4: return launch_bulk_fold<Ty, OP, 4, kBulkRing, WIRE>(p, seg, s);
    case 8: return launch_bulk_fold<Ty, OP, 8, kBulkRing, WIRE>(p, seg, s);
    case 16: return launch_bulk_fold<Ty, OP, 16, kBulkRing, WIRE>(p, seg, s);
    case 32: return launch_bulk_fold<Ty, OP, 32, kBulkRing, WIRE>(p, seg, s);
    case 64: return launch_bulk_fold<Ty, OP, 64, kBulkRing, WIRE>(p, seg, s);
    }
    return launch_bulk_fold<Ty, OP, 0, kBulkRing, WIRE>(p, seg, s);
}

uint64_t tiles_of(uint64_t elems, int esize, int n)
{
    const uint64_t te = (uint64_t)bulk_launch_tile_vectors(n) * (16u / (uint64_t)esize);
    return elems ? (elems + te - 1) / te : 1;
}

}  // namespace

unsigned int* bulk_wait_counters()
{
    constexpr int kMaxDevices = 64;
    static std::atomic<unsigned int*> ptr[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    unsigned int* p = ptr[dev].load(std::memory_order_acquire);
    if (p) return p;
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_bulk_waits) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    ptr[dev].store(static_cast<unsigned int*>(q), std::memory_order_release);  // a racing lookup stores the same
    return static_cast<unsigned int*>(q);
}

BulkParams bulk_params(const RankParams& p)
{
    BulkParams bp{};
    bp.r = p;
    bp.waits = p.waits;
    bp.hold = bulk_debug().hold;
    bp.spin = bulk_debug().spin;
    return bp;
}

bool bulk_eligible(const RankParams& p, int esize)
{
    if (!p.waits || p.n < 2 || p.n > kMaxRanks || !p.vec_ok) return false;
    // every input and output at one 16-byte phase, on element boundaries
    const uintptr_t ph = (uintptr_t)p.in[0] % 16;
    if ((uintptr_t)p.out[0] % 16 != ph || ph % (uintptr_t)esize != 0) return false;
    if (p.nseg != (uint64_t)p.n || p.lo >= p.count) return false;
    // one output per chunk (the two-shot's first shot) past 16 ranks: as for the
    // reduce-scatter, too few threads fold each small tile for one small output
    if (p.owner_only && p.n > 16) return false;
    const uint64_t hi = p.hi < p.count ? p.hi : p.count;
    const uint64_t seg = hi - p.lo < p.C ? hi - p.lo : p.C;
    return tiles_of(seg, esize, p.n) * (uint64_t)p.n <= kMaxGrid;
}

bool bulk_scatter_eligible(const RankParams& p, int esize)
{
    // every input at one 16-byte phase (so part r of every rank is too), every
    // output at one phase, all on element boundaries; up to 16 ranks (beyond,
    // a rank's tile is under 1 KB, too few threads fold each tile and a part
    // has one small output to hide that: 64 ranks ran at 0.71 of the copy peak
    // against 1.10 with per-thread loads)
    if (!p.waits || p.n < 2 || p.n > 16 || !p.vec_ok || p.nseg != (uint64_t)p.n) return false;
    if ((uintptr_t)p.in[0] % (uintptr_t)esize != 0 || (uintptr_t)p.out[0] % (uintptr_t)esize != 0) return false;
    return tiles_of(p.C, esize, p.n) * (uint64_t)p.n <= kMaxGrid;
}

bool bulk_tree_eligible(const RankParams& p, int esize)
{
    if (!p.waits || p.n < 2 || p.nseg != 1 || (p.n > 8 && p.n != 12 && p.n != 16) || !p.vec_ok) return false;
    // every buffer at one 16-byte phase, on element boundaries
    const uintptr_t ph = (uintptr_t)p.in[0] % 16;
    if ((uintptr_t)p.out[0] % 16 != ph || ph % (uintptr_t)esize != 0) return false;
    return tiles_of(p.count, esize, p.n) <= kMaxGrid;
}

template <class Ty, int OP>
cudaError_t launch_oneshot_bulk(const RankParams& p, cudaStream_t s)
{
    return launch_ring<Ty, OP, 0>(p, s);
}

cudaError_t launch_oneshot_wire_bulk(int op, const RankParams& p, cudaStream_t s)
{
    return op == kAvg ? launch_ring<F32T, kAvg, 1>(p, s) : launch_ring<F32T, kSum, 1>(p, s);
}

cudaError_t kernel_binary_version(int* version)
{
    cudaFuncAttributes a{};
    const cudaError_t e = cudaFuncGetAttributes(&a, take_waits_kernel);
    if (e == cudaSuccess) *version = a.binaryVersion;
    return e;
}

cudaError_t take_bulk_timeouts(unsigned int* ran_out, unsigned int* in_flight)
{
    // exchanged on the device, so a count that a kernel adds meanwhile is kept
    // for the next take; the copy below follows the kernel on the same stream
    take_waits_kernel<<<1, 1>>>();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    unsigned int h[2] = {0u, 0u};
    if ((e = cudaMemcpyFromSymbol(h, g_bulk_taken, sizeof h)) != cudaSuccess) return e;
    *ran_out = h[0];
    *in_flight = h[1];
    return cudaSuccess;
}

#define RR_INSTANTIATE(TY, OP) template cudaError_t launch_oneshot_bulk<TY, OP>(const RankParams&, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_INSTANTIATE)
#undef RR_INSTANTIATE

}  // namespace rr
