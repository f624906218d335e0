// rr_noalloc.cu -- the host-buffer all-reduce for callers that cannot
// allocate device memory (rr_allreduce_host_noalloc in include/rr.h).
//
// rr_allreduce_host needs device buffers from its caller.  Some callers have
// none and cannot make any: code that runs while a framework's caching
// allocator holds all of the device's memory, a plug-in given only host
// arrays and a stream, or a latency-critical path that must not call
// cudaMalloc / cudaFree (both may synchronise the device).  This entry point
// stages the ranks' values in one array of device memory that the library
// declares statically below, so the call allocates nothing: its scratch
// exists from the moment the library's device code is loaded on a GPU until
// the process exits.
//
// The array's name, used in host code, is only a host-side stand-in for it;
// its device address is looked up once per device with cudaGetSymbolAddress
// (with that device current) and passed to the copies and the kernel.
#include <atomic>
#include <cstdint>

#include "rr.h"
#include "rr_internal.h"

namespace rr {
rr_status_t record_error(rr_status_t st, const char* why);
void record_stats(const rr_stats_t& s);
}  // namespace rr

using namespace rr;

// The staging area: RR_NOALLOC_MAX_BYTES of device memory, one copy on every
// GPU that loads the library, held until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_staging[RR_NOALLOC_MAX_BYTES];

namespace {

constexpr uint64_t kSlotAlign = 256;  // each rank's slot starts on a 256-byte boundary

// The staging area's device address on the current device, looked up on the
// first call for that device; NULL (with *err set) if the lookup fails.
unsigned char* staging_address(cudaError_t* err)
{
    constexpr int kMaxDevices = 64;
    static std::atomic<unsigned char*> addr[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *err = e != cudaSuccess ? e : cudaErrorInvalidDevice;
        return nullptr;
    }
    unsigned char* p = addr[dev].load(std::memory_order_acquire);
    if (p) return p;
    void* q = nullptr;
    e = cudaGetSymbolAddress(&q, g_noalloc_staging);
    if (e != cudaSuccess) {
        *err = e;
        return nullptr;
    }
    addr[dev].store(static_cast<unsigned char*>(q), std::memory_order_release);  // a racing lookup stores the same
    return static_cast<unsigned char*>(q);
}

uint64_t esize(rr_dtype_t d) { return d == RR_BF16 || d == RR_F16 ? 2u : 4u; }

bool same_phase(void* const* p, int n)
{
    for (int i = 1; i < n; ++i)
        if (((uintptr_t)p[i] & 15u) != ((uintptr_t)p[0] & 15u)) return false;
    return true;
}

}  // namespace

extern "C" rr_status_t rr_allreduce_host_noalloc(void* const* host_bufs, int nranks, size_t count, rr_dtype_t dtype,
                                                 rr_op_t op, rr_algo_t algo, cudaStream_t stream)
{
    if (nranks < 1 || nranks > RR_MAX_RANKS) return record_error(RR_ERR_INVALID_ARG, "nranks must be in 1..64");
    if (dtype != RR_F32 && dtype != RR_BF16 && dtype != RR_I32 && dtype != RR_F16)
        return record_error(RR_ERR_INVALID_ARG, "unknown dtype");
    if (op < RR_SUM || op > RR_PROD) return record_error(RR_ERR_INVALID_ARG, "unknown op");
    if (dtype == RR_I32 && op == RR_AVG) return record_error(RR_ERR_UNSUPPORTED, "AVG is not defined for int32");
    if (algo != RR_ALGO_AUTO && algo != RR_ALGO_ONESHOT)
        return record_error(RR_ERR_UNSUPPORTED, "the no-allocation host all-reduce runs AUTO or ONESHOT");
    if (!host_bufs) return record_error(RR_ERR_INVALID_ARG, "NULL pointer array");
    const int n = nranks;
    const uint64_t es = esize(dtype);
    if (count > RR_NOALLOC_MAX_BYTES / es)
        return record_error(RR_ERR_INVALID_ARG, "the no-allocation host all-reduce stages at most "
                                                "RR_NOALLOC_MAX_BYTES (16 MiB) in all; this call needs more");
    const uint64_t bytes = count * es;
    const uint64_t slot = (bytes + kSlotAlign - 1) / kSlotAlign * kSlotAlign;
    if (slot * (uint64_t)n > RR_NOALLOC_MAX_BYTES)
        return record_error(RR_ERR_INVALID_ARG, "the no-allocation host all-reduce stages at most "
                                                "RR_NOALLOC_MAX_BYTES (16 MiB) in all (each rank's slot rounded "
                                                "up to 256 bytes); this call needs more");
    for (int r = 0; r < n && bytes; ++r) {  // the host buffers are written: non-NULL and disjoint
        if (!host_bufs[r]) return record_error(RR_ERR_INVALID_ARG, "NULL host buffer");
        for (int q = 0; q < r; ++q) {
            const uintptr_t a = (uintptr_t)host_bufs[r], b = (uintptr_t)host_bufs[q];
            if (a < b + bytes && b < a + bytes) return record_error(RR_ERR_INVALID_ARG, "host buffers overlap (or repeat)");
        }
    }
    rr_stats_t st{};
    st.algo = RR_ALGO_ONESHOT;
    st.nranks = n;
    st.bytes_per_rank = bytes;
    if (bytes == 0 || n == 1) {  // nothing to reduce: one rank already holds the result
        record_stats(st);
        return RR_OK;
    }
    cudaError_t e = cudaSuccess;
    unsigned char* base = staging_address(&e);
    if (!base) return record_error(RR_ERR_CUDA, "looking up the static staging area's device address failed");
    void* dev[RR_MAX_RANKS];
    for (int r = 0; r < n; ++r) dev[r] = base + (uint64_t)r * slot;
    for (int r = 0; r < n; ++r)
        if ((e = cudaMemcpyAsync(dev[r], host_bufs[r], bytes, cudaMemcpyHostToDevice, stream)) != cudaSuccess)
            return record_error(RR_ERR_CUDA, "host-to-device copy into the static staging area failed");
    // the one-shot all-reduce of rr_allreduce(ONESHOT) on the staged copies
    RankParams p{};
    for (int r = 0; r < n; ++r) p.in[r] = p.out[r] = dev[r];
    p.n = n;
    p.vec_ok = same_phase(dev, n);
    p.divisor = (float)n;
    p.C = (count + (uint64_t)n - 1) / (uint64_t)n;
    p.count = count;
    p.nseg = (uint64_t)n;
    const uint64_t te = tile_elems(dtype, reduce_vpt(n));
    p.tps = p.C ? (p.C + te - 1) / te : 1;
    p.lo = 0;
    p.hi = UINT64_MAX;
    p.waits = bulk_wait_counters();
    if ((e = launch_rank_kernel(kOneshotRing, dtype, op, p, stream)) != cudaSuccess)
        return record_error(RR_ERR_CUDA, "one-shot all-reduce launch on the static staging area failed");
    for (int r = 0; r < n; ++r)
        if ((e = cudaMemcpyAsync(host_bufs[r], dev[r], bytes, cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
            return record_error(RR_ERR_CUDA, "device-to-host copy from the static staging area failed");
    st.steps = 1;
    st.launches = 1;
    st.bytes_sent_max = (uint64_t)(n - 1) * bytes;
    st.bytes_sent_total = (uint64_t)n * (n - 1) * bytes;
    st.hbm_bytes = 4ull * n * bytes;  // copies in and out, plus the fold's read and write
    record_stats(st);
    return RR_OK;
}
