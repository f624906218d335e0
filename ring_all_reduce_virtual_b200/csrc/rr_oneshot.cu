// rr_oneshot.cu -- the one-shot all-reduce in ring order (and the first shot
// of the two-shot all-reduce).
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "Ring all-reduce and communication volume" and "alpha-beta model"
// (one-shot: every rank reads every peer's buffer directly).
#include "rr_oneshot.cuh"

namespace rr {

namespace {

// ------------------------------------------------ one-shot, ring order
// Segment c = chunk c of every rank buffer; its fold starts on rank c and
// walks the ring (c, c+1, ..., c+N-1 mod N); the result goes to all N
// buffers.  One launch replaces the ring's 2(N-1) steps with the same bits.
// NS > 0: the rank count, fixed at compile time (p.n == NS); 0: runtime.
template <class Ty, int OP, int VPT, int G, int NS, int WIRE = 0>
__global__ void __launch_bounds__(kThreads) oneshot_ring_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const int n = NS > 0 ? NS : p.n;
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
            if (r >= n) r -= n;
            return static_cast<const T*>(p.in[r]) + lo;
        };
        auto out = [&](int o) { return static_cast<T*>(p.out[p.owner_only ? start : o]) + lo; };
        fold_tile<Ty, OP, VPT, G, NS, WIRE>(in, n, out, p.owner_only ? 1 : n, len, tile, p.vec_ok, p.divisor);
    }
}

}  // namespace

template <class Ty, int OP>
cudaError_t launch_oneshot_ring(const RankParams& p, uint64_t work, cudaStream_t s)
{
    if (bulk_eligible(p, (int)sizeof(typename Ty::T))) return launch_oneshot_bulk<Ty, OP>(p, s);
    if (!p.vec_ok && mixed_eligible(p, (int)sizeof(typename Ty::T))) return launch_oneshot_mixed<Ty, OP>(p, s);
    const int n = p.n;
    constexpr int V = kVptReduce;
    switch (n) {
    case 2: return launch_all(oneshot_ring_kernel<Ty, OP, V, 1, 2>, p, work, s);
    case 3: return launch_all(oneshot_ring_kernel<Ty, OP, V, 2, 3>, p, work, s);
    case 4: return launch_all(oneshot_ring_kernel<Ty, OP, V, 3, 4>, p, work, s);
    case 8: return launch_all(oneshot_ring_kernel<Ty, OP, V, 7, 8>, p, work, s);
    case 16: return launch_all(oneshot_ring_kernel<Ty, OP, V, kGroup, 16>, p, work, s);
    }
    return launch_all(oneshot_ring_kernel<Ty, OP, V, kGroup, 0>, p, work, s);
}

// The bf16-wire one-shot (fp32 buffers, SUM or AVG, any rank count; the
// counts 2, 4, 8 and 16 fixed at compile time, as for the plain one-shot).
template <int OP>
cudaError_t launch_oneshot_wire_op(const RankParams& p, uint64_t work, cudaStream_t s)
{
    constexpr int V = kVptReduce;
    switch (p.n) {
    case 2: return launch_all(oneshot_ring_kernel<F32T, OP, V, 1, 2, 1>, p, work, s);
    case 4: return launch_all(oneshot_ring_kernel<F32T, OP, V, 3, 4, 1>, p, work, s);
    case 8: return launch_all(oneshot_ring_kernel<F32T, OP, V, 7, 8, 1>, p, work, s);
    case 16: return launch_all(oneshot_ring_kernel<F32T, OP, V, kGroup, 16, 1>, p, work, s);
    }
    return launch_all(oneshot_ring_kernel<F32T, OP, V, kGroup, 0, 1>, p, work, s);
}

cudaError_t launch_oneshot_wire(int op, const RankParams& p, uint64_t work, cudaStream_t s)
{
    if (bulk_eligible(p, (int)sizeof(float))) return launch_oneshot_wire_bulk(op, p, s);
    if (!p.vec_ok && mixed_eligible(p, (int)sizeof(float))) return launch_oneshot_wire_mixed(op, p, s);
    return op == kAvg ? launch_oneshot_wire_op<kAvg>(p, work, s) : launch_oneshot_wire_op<kSum>(p, work, s);
}

#define RR_INSTANTIATE(TY, OP) \
    template cudaError_t launch_oneshot_ring<TY, OP>(const RankParams&, uint64_t, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_INSTANTIATE)
#undef RR_INSTANTIATE

}  // namespace rr
