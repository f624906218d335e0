// rr_chain.cu -- the ring, double-ring and tree schedules, each in one
// launch.
//
// The ring's reduce-scatter step s has rank r fold the chunk it receives from
// its left neighbour, k = (r - s - 1) mod N, into its own copy; the
// all-gather step s has rank r overwrite chunk (r - s) mod N with its left
// neighbour's copy ([P4] "Ring all-reduce and communication volume",
// ring_allreduce.py; [P3] section 3).  Followed along one chunk k, the
// schedule is a chain: reduce-scatter step s is done by rank k + s + 1 on the
// partial rank k + s wrote at step s - 1, the chunk is complete on rank
// k - 1, and all-gather step s has rank k + s copy it from rank k + s - 1.
// Different chunks -- and different tiles of one chunk -- never read each
// other's elements.  So a CTA takes one tile of one chunk through all 2(N-1)
// steps, in order, reading the neighbour's copy from memory and writing its
// own at every step exactly as the per-step launches do (the same values in
// the same buffers, the same bytes), and every thread touches the same
// elements at every step, so it only ever reads what it wrote itself: no CTA
// waits for another, and 2(N-1) launches become one.
//
// The double ring ([P3] section 6) is two such sets of chains: the first half
// clockwise, the second half counter-clockwise (each step's partial comes
// from the right neighbour).  The tree schedule ([P3] section 6) chains the
// same way along one tile of the whole buffer: the pairwise reduce levels,
// then the broadcast levels, each pair in turn.
#include "rr_launch.cuh"

namespace rr {

namespace {

constexpr int kChainVpt = 2;  // 16-byte vectors per thread per tile (about 30 registers each)

// The chains' 16-byte accesses: streaming hints (CACHE 0, evict first), or
// default caching (CACHE 1).  Every chain reads back only what its own thread
// wrote, so either is coherent.  Measured per schedule at 3 / 8 / 24 ranks x
// 256 MiB fp32, streaming / cached: ring 0.273 / 0.728 / 3.34 against 0.290 /
// 0.782 / 3.30 ms; tree 0.269 / 0.810 / 2.83 against 0.243 / 0.719 / 2.58 ms;
// bf16-wire ring 0.291 / 0.713 / 3.37 against 0.283 / 0.703 / 3.34 ms.  So
// the plain ring streams, the tree and the wire ring cache.
template <int CACHE>
__device__ __forceinline__ uint4 chain_ld(const void* p)
{
    if constexpr (CACHE) return *reinterpret_cast<const uint4*>(p);
    else return ldv(p);
}
template <int CACHE>
__device__ __forceinline__ void chain_st(void* p, const uint4& v)
{
    if constexpr (CACHE) *reinterpret_cast<uint4*>(p) = v;
    else stv(p, v);
}
constexpr uint64_t kChainTileVecs = (uint64_t)kThreads * kChainVpt;

// The elements one thread owns in one tile of a segment of `len` elements
// whose copies all start at the same 16-byte phase: up to kChainVpt whole
// vectors, and in tile 0 one element of the scalar head or tail.  A thread
// keeps these at every step of the chain.
template <class Ty>
struct ChainLanes {
    uint64_t vec[kChainVpt];  // element offset of each owned vector
    bool ok[kChainVpt];
    uint64_t one;             // owned scalar element
    bool has_one;

    __device__ __forceinline__ ChainLanes(const typename Ty::T* first, uint64_t len, uint64_t tile)
    {
        constexpr int L = Ty::L;
        uint64_t head = (uint64_t)((L - phase_of(first, L)) & (L - 1));
        if (head > len) head = len;
        const uint64_t nv = (len - head) / L, tail = len - head - nv * L;
        const uint64_t tid = threadIdx.x;
        has_one = tile == 0 && tid < head + tail;
        one = tid < head ? tid : head + nv * L + (tid - head);
#pragma unroll
        for (int u = 0; u < kChainVpt; ++u) {
            const uint64_t v = tile * kChainTileVecs + (uint64_t)u * kThreads + tid;
            ok[u] = v < nv;
            vec[u] = head + v * L;
        }
    }
};

// One reduce-scatter step on a thread's lanes: dst = src op dst (the
// arriving partial on the left), then AVG's division and the wire rounding
// where the step completes the chunk.  WIRE: 0 none, 1 completing step, 2
// partial step (see wire_in / wire_out).
template <class Ty, int OP, int WIRE, int CACHE>
__device__ __forceinline__ void chain_fold(const ChainLanes<Ty>& ln, const typename Ty::T* src, typename Ty::T* dst,
                                           float divisor)
{
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;
    if (ln.has_one) {
        Acc a = apply<OP>(wire_in<WIRE>(Ty::ld1(src + ln.one)), Ty::ld1(dst + ln.one));
        Ty::st1(dst + ln.one, wire_out<WIRE>(finish<OP>(a, divisor)));
    }
    uint4 x[kChainVpt], y[kChainVpt];
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) {
            x[u] = chain_ld<CACHE>(src + ln.vec[u]);
            y[u] = chain_ld<CACHE>(dst + ln.vec[u]);
        }
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) {
            Acc a[L], b[L];
            Ty::unpack(x[u], a);
            Ty::unpack(y[u], b);
#pragma unroll
            for (int l = 0; l < L; ++l) a[l] = wire_out<WIRE>(finish<OP>(apply<OP>(wire_in<WIRE>(a[l]), b[l]), divisor));
            chain_st<CACHE>(dst + ln.vec[u], Ty::pack(a));
        }
}

// The next reduce-scatter step's own operand (the receiving rank's copy,
// which nothing writes before that step) copied by cp.async into this
// thread's shared-memory slots, so that the step waits only for the
// neighbour's partial.  Each thread reads only the slots it filled, after its
// own cp.async.wait_group: no barrier.  Used by the bf16-wire ring, whose
// rounding steps lengthen each step: measured at 3 / 8 / 24 / 48 ranks x
// 256 MiB, 0.317 / 0.818 / 3.53 / 7.86 ms without and 0.291 / 0.711 / 3.37 /
// 7.47 ms with it; the plain ring, bound by the read of the partial it has
// just stored, moved by -1 to +2 % and keeps its loads.
template <class Ty>
__device__ __forceinline__ void chain_stage(const ChainLanes<Ty>& ln, const typename Ty::T* own, uint4* slot)
{
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u])
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                             (uint32_t)__cvta_generic_to_shared(slot + u * kThreads + threadIdx.x)),
                         "l"(own + ln.vec[u])
                         : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// chain_fold with the own operand taken from the stage slots.
template <class Ty, int OP, int WIRE, int CACHE>
__device__ __forceinline__ void chain_fold_staged(const ChainLanes<Ty>& ln, const typename Ty::T* src,
                                                  typename Ty::T* dst, const uint4* slot, float divisor)
{
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;
    if (ln.has_one) {
        Acc a = apply<OP>(wire_in<WIRE>(Ty::ld1(src + ln.one)), Ty::ld1(dst + ln.one));
        Ty::st1(dst + ln.one, wire_out<WIRE>(finish<OP>(a, divisor)));
    }
    uint4 x[kChainVpt];
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) x[u] = chain_ld<CACHE>(src + ln.vec[u]);
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) {
            Acc a[L], b[L];
            Ty::unpack(x[u], a);
            Ty::unpack(slot[u * kThreads + threadIdx.x], b);
#pragma unroll
            for (int l = 0; l < L; ++l) a[l] = wire_out<WIRE>(finish<OP>(apply<OP>(wire_in<WIRE>(a[l]), b[l]), divisor));
            chain_st<CACHE>(dst + ln.vec[u], Ty::pack(a));
        }
}

// One all-gather (or broadcast) step on a thread's lanes: dst = src, bits.
template <class Ty, int CACHE>
__device__ __forceinline__ void chain_copy(const ChainLanes<Ty>& ln, const typename Ty::T* src, typename Ty::T* dst)
{
    if (ln.has_one) dst[ln.one] = src[ln.one];
    uint4 x[kChainVpt];
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) x[u] = chain_ld<CACHE>(src + ln.vec[u]);
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) chain_st<CACHE>(dst + ln.vec[u], x[u]);
}

// One tree reduce step on a thread's lanes: out = a op b (a on the left).
template <class Ty, int OP, int CACHE>
__device__ __forceinline__ void tree_fold_pair(const ChainLanes<Ty>& ln, const typename Ty::T* a_, const typename Ty::T* b_,
                                               typename Ty::T* out, float divisor)
{
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;
    if (ln.has_one) Ty::st1(out + ln.one, finish<OP>(apply<OP>(Ty::ld1(a_ + ln.one), Ty::ld1(b_ + ln.one)), divisor));
    uint4 x[kChainVpt], y[kChainVpt];
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) {
            x[u] = chain_ld<CACHE>(a_ + ln.vec[u]);
            y[u] = chain_ld<CACHE>(b_ + ln.vec[u]);
        }
#pragma unroll
    for (int u = 0; u < kChainVpt; ++u)
        if (ln.ok[u]) {
            Acc a[L], b[L];
            Ty::unpack(x[u], a);
            Ty::unpack(y[u], b);
#pragma unroll
            for (int l = 0; l < L; ++l) a[l] = finish<OP>(apply<OP>(a[l], b[l]), divisor);
            chain_st<CACHE>(out + ln.vec[u], Ty::pack(a));
        }
}

// Ring work item w -> (direction, chunk k, tile) and the chunk's elements
// [lo, lo + len); false for an empty chunk.
__device__ __forceinline__ bool chain_segment(const ChainParams& p, uint64_t w, int& dir, int& k, uint64_t& tile,
                                              uint64_t& lo, uint64_t& len)
{
    const uint64_t per_half = (uint64_t)p.n * p.tps;
    const int h = (int)(w / per_half);
    const uint64_t rem = w - (uint64_t)h * per_half;
    k = (int)(rem / p.tps);
    tile = rem - (uint64_t)k * p.tps;
    const uint64_t base = h == 0 ? 0 : p.H, span = h == 0 ? p.H : p.count - p.H;
    const uint64_t c = p.C[h], c_lo = (uint64_t)k * c;
    if (c_lo >= span) return false;
    lo = base + c_lo;
    len = c < span - c_lo ? c : span - c_lo;
    dir = h == 0 ? 1 : -1;
    return true;
}

__device__ __forceinline__ int wrap(int r, int n) { return r < 0 ? r + n : (r >= n ? r - n : r); }

template <class Ty, int OP, bool WIRE>
__global__ void __launch_bounds__(kThreads) ring_chain_kernel(const __grid_constant__ ChainParams p)
{
    using T = typename Ty::T;
    constexpr int OPP = OP == kAvg ? kSum : OP;  // partial steps: AVG divides only where a chunk completes
    const int n = p.n;
    const uint64_t total = (uint64_t)p.nhalf * p.n * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        int dir, k;
        uint64_t tile, lo, len;
        if (!chain_segment(p, w, dir, k, tile, lo, len)) continue;
        const ChainLanes<Ty> ln(static_cast<const T*>(p.buf[k]) + lo, len, tile);
        if (!ln.has_one && !ln.ok[0]) continue;
        // reduce-scatter step s: rank k + dir (s + 1) folds its neighbour's partial into its copy
        if constexpr (WIRE) {
            __shared__ uint4 stage[2][kChainVpt * kThreads];
            chain_stage<Ty>(ln, static_cast<const T*>(p.buf[wrap(k + dir, n)]) + lo, stage[0]);
#pragma unroll 1
            for (int s = 0; s < n - 1; ++s) {
                const int r = wrap(k + dir * (s + 1), n), from = wrap(r - dir, n);
                const T* src = static_cast<const T*>(p.buf[from]) + lo;
                T* dst = static_cast<T*>(p.buf[r]) + lo;
                if (s + 1 < n - 1) {
                    chain_stage<Ty>(ln, static_cast<const T*>(p.buf[wrap(r + dir, n)]) + lo, stage[(s + 1) & 1]);
                    asm volatile("cp.async.wait_group 1;" ::: "memory");
                } else {
                    asm volatile("cp.async.wait_group 0;" ::: "memory");
                }
                if (s == n - 2) chain_fold_staged<Ty, OP, 1, 1>(ln, src, dst, stage[s & 1], p.divisor);
                else chain_fold_staged<Ty, OPP, 2, 1>(ln, src, dst, stage[s & 1], p.divisor);
            }
        } else {
#pragma unroll 1
            for (int s = 0; s < n - 1; ++s) {
                const int r = wrap(k + dir * (s + 1), n), from = wrap(r - dir, n);
                const T* src = static_cast<const T*>(p.buf[from]) + lo;
                T* dst = static_cast<T*>(p.buf[r]) + lo;
                if (s == n - 2) chain_fold<Ty, OP, 0, 0>(ln, src, dst, p.divisor);
                else chain_fold<Ty, OPP, 0, 0>(ln, src, dst, p.divisor);
            }
        }
        // all-gather step s: rank k + dir s copies the finished chunk from its neighbour
#pragma unroll 1
        for (int s = 0; s < n - 1; ++s) {
            const int r = wrap(k + dir * s, n), from = wrap(r - dir, n);
            chain_copy<Ty, WIRE ? 1 : 0>(ln, static_cast<const T*>(p.buf[from]) + lo, static_cast<T*>(p.buf[r]) + lo);
        }
    }
}

template <class Ty, int OP>
__global__ void __launch_bounds__(kThreads) tree_chain_kernel(const __grid_constant__ ChainParams p)
{
    using T = typename Ty::T;
    constexpr int OPP = OP == kAvg ? kSum : OP;
    const int n = p.n;
    int levels = 0;
    while ((1 << levels) < n) ++levels;
    for (uint64_t tile = blockIdx.x; tile < p.tps; tile += gridDim.x) {
        const ChainLanes<Ty> ln(static_cast<const T*>(p.buf[0]), p.count, tile);
        if (!ln.has_one && !ln.ok[0]) continue;
#pragma unroll 1
        for (int l = 0; l < levels; ++l) {  // reduce: x_a <- x_a op x_{a+h}; AVG divides at the top level
            const int h = 1 << l;
#pragma unroll 1
            for (int a = 0; a + h < n; a += 2 * h) {
                // chain_fold folds src into dst with src on the left: here x_a is the left operand
                const T* xa = static_cast<const T*>(p.buf[a]);
                T* xb = static_cast<T*>(p.buf[a + h]);
                if (l == levels - 1) tree_fold_pair<Ty, OP, 1>(ln, xa, xb, static_cast<T*>(p.buf[a]), p.divisor);
                else tree_fold_pair<Ty, OPP, 1>(ln, xa, xb, static_cast<T*>(p.buf[a]), p.divisor);
            }
        }
#pragma unroll 1
        for (int l = levels - 1; l >= 0; --l) {  // broadcast: x_{a+h} <- x_a
            const int h = 1 << l;
#pragma unroll 1
            for (int a = 0; a + h < n; a += 2 * h)
                chain_copy<Ty, 1>(ln, static_cast<const T*>(p.buf[a]), static_cast<T*>(p.buf[a + h]));
        }
    }
}

}  // namespace

uint64_t chain_tile_elems(int dtype) { return kChainTileVecs * (dtype == kBF16 || dtype == kF16 ? 8u : 4u); }

cudaError_t launch_ring_chain(int dtype, int op, bool wire, const ChainParams& p, cudaStream_t s)
{
    const uint64_t work = (uint64_t)p.nhalf * p.n * p.tps;
    if (wire) {
        if (dtype != kF32) return cudaErrorInvalidValue;
        return op == kAvg ? launch_all(ring_chain_kernel<F32T, kAvg, true>, p, work, s)
                          : launch_all(ring_chain_kernel<F32T, kSum, true>, p, work, s);
    }
    return with_type(dtype, op, [&]<class Ty, int OP>() { return launch_all(ring_chain_kernel<Ty, OP, false>, p, work, s); });
}

cudaError_t launch_tree_chain(int dtype, int op, const ChainParams& p, cudaStream_t s)
{
    return with_type(dtype, op, [&]<class Ty, int OP>() { return launch_all(tree_chain_kernel<Ty, OP>, p, p.tps, s); });
}

}  // namespace rr
