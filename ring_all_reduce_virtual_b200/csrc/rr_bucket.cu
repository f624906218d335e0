// rr_bucket.cu -- DDP-style gradient buckets: pack (gradients -> fp32
// bucket), unpack (fp32 bucket -> gradients, with AVG's division and one
// rounding) and the fused bucket sync that does pack + ring-order all-reduce
// + unpack in one pass over the gradients.
//
// Sources: [P1] "How all-reduce keeps every card identical" (mhpq.cn),
// s5.1-5.2 (DDP buckets, bucket_cap_mb = 25) and s5.3 (reduce low-precision
// gradients in fp32); [P2] "AllReduce from principle to tuning" (xxqk.cn),
// s3.3 (gradients fill buckets in order; a full bucket triggers its
// all-reduce); [P3] "Training gradient sync and collective communication"
// (geek-doc.cn), section 5 (bucketing hides the per-message latency).
#include "rr_bulk.cuh"

namespace rr {

namespace {

constexpr int kUnitsPerThread = 4;

// Four elements of a gradient or bucket type as raw bits: one 16-byte vector
// of fp32, or 8 bytes of bf16.  Pack and unpack move quads, so both sides of
// a conversion are read and written with whole, contiguous warp accesses
// (lane i touches quad i of the warp's run).
template <class X>
struct Quad;

template <>
struct Quad<F32T> {
    using R = uint4;
    __device__ static __forceinline__ R ld(const float* p) { return ldv(p); }
    __device__ static __forceinline__ void st(float* p, const R& r) { stv(p, r); }
    __device__ static __forceinline__ void to_f(const R& r, float (&a)[4]) { F32T::unpack(r, a); }
    __device__ static __forceinline__ R from_f(const float (&a)[4]) { return F32T::pack(a); }
    // The four elements that start d elements into the aligned window lo:hi.
    __device__ static __forceinline__ R shift(const R& lo, const R& hi, int d)
    {
        switch (d) {
        case 1: return make_uint4(lo.y, lo.z, lo.w, hi.x);
        case 2: return make_uint4(lo.z, lo.w, hi.x, hi.y);
        case 3: return make_uint4(lo.w, hi.x, hi.y, hi.z);
        }
        return lo;
    }
};

// The 16-bit types (bf16, fp16): a quad is 8 bytes, two packed pairs.
template <class X>
struct Quad16 {
    using R = uint2;
    __device__ static __forceinline__ R ld(const uint16_t* p) { return __ldcs(reinterpret_cast<const uint2*>(p)); }
    __device__ static __forceinline__ void st(uint16_t* p, const R& r) { __stcs(reinterpret_cast<uint2*>(p), r); }
    __device__ static __forceinline__ void to_f(const R& r, float (&a)[4])
    {
        X::unpack2(r.x, a[0], a[1]);
        X::unpack2(r.y, a[2], a[3]);
    }
    __device__ static __forceinline__ R from_f(const float (&a)[4])
    {
        return make_uint2(X::pack2(a[0], a[1]), X::pack2(a[2], a[3]));
    }
    // The four elements that start d elements into the aligned window lo:hi
    // (element j is the low half of word j / 2 when j is even).
    __device__ static __forceinline__ R shift(const R& lo, const R& hi, int d)
    {
        const uint32_t w0 = d >= 2 ? lo.y : lo.x, w1 = d >= 2 ? hi.x : lo.y, w2 = d >= 2 ? hi.y : hi.x;
        if (d & 1) return make_uint2(__funnelshift_r(w0, w1, 16), __funnelshift_r(w1, w2, 16));
        return make_uint2(w0, w1);
    }
};

template <>
struct Quad<BF16T> : Quad16<BF16T> {};

template <>
struct Quad<F16T> : Quad16<F16T> {};

// The quads of one tile of a conversion (see convert_tile) whose source
// quads are in step with the destination's: one aligned load per quad, Q per
// thread all issued before the first one is used.
template <class In, class Out, int OP, int Q>
__device__ __forceinline__ void convert_quads(const typename In::T* s0, typename Out::T* dst, uint64_t head, uint64_t nq,
                                              uint64_t tile, float divisor)
{
    constexpr uint64_t TQ = (uint64_t)kThreads * Q;
    constexpr int QP = 4;  // quads per pass: 64 bytes of fp32 on the wider side
    static_assert(Q % QP == 0, "whole passes");
    const uint64_t tid = threadIdx.x;
#pragma unroll
    for (int pass = 0; pass < Q / QP; ++pass) {
        typename Quad<In>::R raw[QP];
#pragma unroll
        for (int k = 0; k < QP; ++k) {
            const uint64_t q = tile * TQ + (uint64_t)(pass * QP + k) * kThreads + tid;
            if (q < nq) raw[k] = Quad<In>::ld(s0 + q * 4);
        }
#pragma unroll
        for (int k = 0; k < QP; ++k) {
            const uint64_t q = tile * TQ + (uint64_t)(pass * QP + k) * kThreads + tid;
            if (q >= nq) continue;
            float a[4];
            Quad<In>::to_f(raw[k], a);
#pragma unroll
            for (int l = 0; l < 4; ++l) a[l] = finish<OP>(a[l], divisor);
            Quad<Out>::st(dst + head + q * 4, Quad<Out>::from_f(a));
        }
    }
}

// The same when the source quads are d = 1..3 elements out of step (fp32
// sources): the tile's source quads (and the one after, which holds the last
// few elements) are copied aligned by cp.async -- one copy per quad, all in
// flight, none through registers -- into shared memory, and each destination
// quad reads the two stage quads it straddles and shifts them in registers,
// so no global load is issued twice.  Every thread of the CTA takes part (the
// tile is the CTA's).  Measured on the unpack of 2-8 ranks x 64 Mi bf16
// parameters 1 and 2 elements out of phase: 0.93-1.06 of the copy peak,
// against 0.82-0.97 with the stage filled through registers.
template <class In, class Out, int OP, int Q>
__device__ __forceinline__ void convert_quads_staged(const typename In::T* s0, typename Out::T* dst, uint64_t head,
                                                     uint64_t nq, uint64_t tile, int d, float divisor)
{
    using R = typename Quad<In>::R;
    static_assert(sizeof(R) == 16, "16-byte source quads (fp32): the 16-bit sources take convert_quads_shfl");
    constexpr uint32_t TQ = (uint32_t)kThreads * Q;
    __shared__ R stage[TQ + 1];
    const uint64_t q0 = tile * TQ;
    if (q0 >= nq) return;
    const uint32_t nqt = nq - q0 < TQ ? (uint32_t)(nq - q0) : TQ;  // destination quads of this tile
    // global -> shared without passing through registers, all of the
    // thread's copies in flight
#pragma unroll
    for (int k = 0; k <= Q; ++k) {
        const uint32_t i = (uint32_t)k * kThreads + threadIdx.x;
        if (i <= nqt)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(&stage[i])),
                         "l"(s0 + (q0 + i) * 4)
                         : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
#pragma unroll
    for (int k = 0; k < Q; ++k) {
        const uint32_t i = (uint32_t)k * kThreads + threadIdx.x;
        if (i >= nqt) continue;
        float a[4];
        Quad<In>::to_f(Quad<In>::shift(stage[i], stage[i + 1], d), a);  // two aligned stage reads, shifted
#pragma unroll
        for (int l = 0; l < 4; ++l) a[l] = finish<OP>(a[l], divisor);
        Quad<Out>::st(dst + head + (q0 + i) * 4, Quad<Out>::from_f(a));
    }
    __syncthreads();  // the stage is free for the CTA's next tile
}

// The same with the shift done across lanes instead of through shared
// memory: each warp takes a run of 32 * Q destination quads (32 consecutive
// quads per access, all Q loads in flight), and a lane takes the source quad
// after its own from lane + 1 by warp shuffle -- lane 31 from lane 0 of the
// next access, or for the warp's last access from one more load.
template <class In, class Out, int OP, int Q>
__device__ __forceinline__ void convert_quads_shfl(const typename In::T* s0, typename Out::T* dst, uint64_t head,
                                                   uint64_t nq, uint64_t tile, int d, float divisor)
{
    using R = typename Quad<In>::R;
    constexpr uint32_t TQ = (uint32_t)kThreads * Q;
    constexpr int W = sizeof(R) / 4;  // 32-bit words per quad
    const uint64_t q0 = tile * TQ;
    if (q0 >= nq) return;
    const uint32_t nqt = nq - q0 < TQ ? (uint32_t)(nq - q0) : TQ;  // destination quads of this tile
    const uint32_t lane = threadIdx.x & 31u, b = (threadIdx.x >> 5) * 32u * Q;  // the warp's first quad
    R cur[Q], after{};
#pragma unroll
    for (int k = 0; k < Q; ++k) {
        const uint32_t i = b + (uint32_t)k * 32u + lane;
        cur[k] = R{};
        if (i <= nqt) cur[k] = Quad<In>::ld(s0 + (q0 + i) * 4);
    }
    const uint32_t ia = b + 32u * Q;  // the quad after the warp's run
    if (lane == 31u && ia <= nqt) after = Quad<In>::ld(s0 + (q0 + ia) * 4);
#pragma unroll
    for (int k = 0; k < Q; ++k) {
        R nb;
        const R& nx = k + 1 < Q ? cur[k + 1 < Q ? k + 1 : k] : after;
        uint32_t* o = reinterpret_cast<uint32_t*>(&nb);
        const uint32_t* c = reinterpret_cast<const uint32_t*>(&cur[k]);
        const uint32_t* x = reinterpret_cast<const uint32_t*>(&nx);
#pragma unroll
        for (int w = 0; w < W; ++w) {
            const uint32_t up = __shfl_sync(0xffffffffu, c[w], (lane + 1u) & 31u);
            const uint32_t first = __shfl_sync(0xffffffffu, x[w], 0);
            o[w] = lane == 31u ? (k + 1 < Q ? first : x[w]) : up;
        }
        const uint32_t i = b + (uint32_t)k * 32u + lane;
        if (i >= nqt) continue;
        float a[4];
        Quad<In>::to_f(Quad<In>::shift(cur[k], nb, d), a);
#pragma unroll
        for (int l = 0; l < 4; ++l) a[l] = finish<OP>(a[l], divisor);
        Quad<Out>::st(dst + head + (q0 + i) * 4, Quad<Out>::from_f(a));
    }
}

// Convert one tile of a segment from In's element type to Out's, dividing by
// `divisor` first when OP is AVG.  A tile is kThreads * Q quads, Q chosen so
// that it covers kThreads * kUnitsPerThread 16-byte vectors of the narrower
// type (bucket_tile_elems).  The quads are aligned to the destination: after
// a scalar head up to dst's first quad boundary, every quad is one aligned
// store, and its source elements -- which start d = (phase of src - phase of
// dst) mod 4 elements into an aligned source quad -- are read from that quad
// and, when d > 0, the next one, through shared memory (convert_quads_staged).
// Every source quad loaded holds at least one element of the segment, so no
// load reaches past the aligned block of the segment's last element (nor
// before the block of its first).  Tile 0 also does the head and the tail
// (< 4 elements each).  Every thread of the CTA calls this for the same tile.
template <class In, class Out, int OP, int Q = kUnitsPerThread * (In::L > Out::L ? In::L : Out::L) / 4>
__device__ __forceinline__ void convert_tile(const typename In::T* src, typename Out::T* dst, uint64_t len,
                                             uint64_t tile, float divisor)
{
    const int tid = threadIdx.x;
    const int pd = phase_of(dst, 4);
    const int d = (phase_of(src, 4) - pd) & 3;
    uint64_t head = (uint64_t)((4 - pd) & 3);
    if (head > len) head = len;
    const uint64_t nq = (len - head) / 4;
    const uint64_t tail = len - head - nq * 4;
    if (tile == 0 && (uint64_t)tid < head + tail) {
        const uint64_t e = (uint64_t)tid < head ? (uint64_t)tid : head + nq * 4 + ((uint64_t)tid - head);
        Out::st1(dst + e, finish<OP>((float)In::ld1(src + e), divisor));
    }
    // the aligned source quad under dst's first quad (d elements before src + head)
    const auto* s0 = reinterpret_cast<const typename In::T*>(reinterpret_cast<uintptr_t>(src + head) -
                                                              (uintptr_t)d * sizeof(typename In::T));
    // shifted quads of a 16-bit source (the pack) by warp shuffle, of an fp32
    // source (the unpack) through shared memory: measured on 8 x 64 Mi bf16
    // parameters 1 and 2 elements out of phase, the shuffles ran the pack at
    // 1.005 of the copy peak against 1.002 with a register-filled stage, but
    // the unpack at 0.90 against 0.97 (holding eight 16-byte quads a thread
    // took 74 registers), and 1.06 with the cp.async stage
    if (d == 0) convert_quads<In, Out, OP, Q>(s0, dst, head, nq, tile, divisor);
    else if constexpr (sizeof(typename Quad<In>::R) == 8) convert_quads_shfl<In, Out, OP, Q>(s0, dst, head, nq, tile, d, divisor);
    else convert_quads_staged<In, Out, OP, Q>(s0, dst, head, nq, tile, d, divisor);
}

// The segment owning work item w: the last s with prefix[s] <= w (segments
// without tiles have prefix[s] == prefix[s + 1] and are never returned).
__device__ __forceinline__ int find_segment(const uint64_t* prefix, int nseg, uint64_t w)
{
    int lo = 0, hi = nseg;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= w) lo = mid;
        else hi = mid;
    }
    return lo;
}

// Work item w of a pack/unpack launch -> (tensor t, rank r, tile).
__device__ __forceinline__ void copy_item(const BucketCopyParams& p, uint64_t w, uint64_t& t, uint64_t& r,
                                          uint64_t& tile)
{
    t = (uint64_t)find_segment(p.tile0, p.nt, w);
    const uint64_t local = w - p.tile0[t];
    const uint64_t tiles = (p.tile0[t + 1] - p.tile0[t]) / (uint64_t)p.n;
    r = local / tiles;
    tile = local - r * tiles;
}

// Pack: segment (t, r) copies rank r's tensor t into rank r's fp32 bucket at
// the tensor's offset (exact widening).
template <class G>
__global__ void __launch_bounds__(kThreads) bucket_pack_kernel(const __grid_constant__ BucketCopyParams p)
{
    const uint64_t total = p.tile0[p.nt];
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        uint64_t t, r, tile;
        copy_item(p, w, t, r, tile);
        const uint64_t s = t * (uint64_t)p.n + r;
        const auto* src = static_cast<const typename G::T*>(p.grad[s]);
        float* dst = static_cast<float*>(p.bucket[r]) + p.toff[t];
        convert_tile<G, F32T, kSum>(src, dst, p.tlen[t], tile, 1.0f);
    }
}

// Unpack: segment (t, r) writes round(bucket[r][toff + j] / N) (AVG) or
// round(bucket[r][toff + j]) (SUM) into rank r's tensor t.
template <class G, int OP>
__global__ void __launch_bounds__(kThreads) bucket_unpack_kernel(const __grid_constant__ BucketCopyParams p)
{
    const uint64_t total = p.tile0[p.nt];
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        uint64_t t, r, tile;
        copy_item(p, w, t, r, tile);
        const uint64_t s = t * (uint64_t)p.n + r;
        const float* src = static_cast<const float*>(p.bucket[r]) + p.toff[t];
        auto* dst = static_cast<typename G::T*>(const_cast<void*>(p.grad[s]));
        convert_tile<F32T, G, OP>(src, dst, p.tlen[t], tile, p.divisor);
    }
}

// Fused bucket sync: segment = a run of one tensor inside one chunk c of the
// bucket's flat index; every rank's copy is read once, folded in fp32 in ring
// order from rank c, divided (AVG), rounded once and written back to every
// rank.  Same bits as pack -> one-shot all-reduce (SUM) -> unpack.
template <class G, int OP, int VPT, int GR, int NS>
__global__ void __launch_bounds__(kThreads) bucket_fold_kernel(const __grid_constant__ BucketFoldParams p)
{
    using T = typename G::T;
    const uint64_t total = p.tile0[p.nseg];
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const int s = find_segment(p.tile0, p.nseg, w);
        const uint64_t tile = w - p.tile0[s];
        const BucketSeg& sg = p.seg[s];
        const int n = NS > 0 ? NS : p.n;
        const int base = (int)sg.t * n;
        const int start = (int)sg.c;
        auto in = [&](int j) {
            int r = start + j;
            if (r >= n) r -= n;
            return static_cast<const T*>(p.grad[base + r]) + sg.off;
        };
        auto out = [&](int o) { return static_cast<T*>(p.grad[base + o]) + sg.off; };
        fold_tile<G, OP, VPT, GR, NS>(in, n, out, n, sg.len, tile, p.vec_ok, p.divisor);
    }
}

// The fused bucket sync with its tiles staged by bulk async copies (the
// fold of rr_bulk.cuh: one elected thread copies the N ranks' tiles into
// shared memory behind a bounded mbarrier wait, the CTA folds them in ring
// order, the thread bulk-stores the result to every rank).  A segment starts
// at any element, so tile 0 folds the elements before the segment's first
// 16-byte boundary and after its last whole vector with plain loads, and the
// bulk copies move the whole vectors between.  Needs every rank's copy of a
// tensor at the same address modulo 16 (vec_ok) and 2 or more ranks (2, 4, 8
// and 16 fixed at compile time, the others a kernel argument).
struct BucketBulkParams {
    BucketFoldParams f;  // tile0 counts bulk tiles (bucket_bulk_tile_elems)
    unsigned int* waits; // as BulkParams (rr_bulk.cuh): the wait counters, the test hook, the bound
    uint32_t hold;
    uint32_t spin;
    uint32_t tv;         // vectors per rank per tile (kernels whose rank count is not fixed)
};
static_assert(sizeof(BucketBulkParams) <= 32764, "BucketBulkParams too large");

template <class G, int OP, int NS>
__global__ void __launch_bounds__(kThreads) bucket_bulk_kernel(const __grid_constant__ BucketBulkParams bp)
{
    using T = typename G::T;
    using Acc = typename G::Acc;
    constexpr int L = G::L;
    // When launched as a programmatic dependent of the stream's previous
    // kernel (direct bucket-sync calls): wait for that kernel and its memory
    // before touching the gradients, and let the next sync's CTAs be
    // scheduled while this grid drains.  Launched plainly, both are no-ops.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const BucketFoldParams& p = bp.f;
    const int n = NS > 0 ? NS : p.n;
    const uint32_t TV = NS > 0 ? bulk_smem<NS>() / (NS > 0 ? NS : 1) / 16 : bp.tv;  // vectors per rank per tile
    extern __shared__ __align__(128) uint4 sm[];       // [n][TV]: slot j holds rank (c + j) mod N
    __shared__ __align__(8) uint64_t bar;

    const uint64_t w = blockIdx.x;
    const int s = find_segment(p.tile0, p.nseg, w);
    const uint64_t tile = w - p.tile0[s];
    const BucketSeg& sg = p.seg[s];
    const int base = (int)sg.t * n;
    const int start = (int)sg.c;
    auto in = [&](int j) {
        int r = start + j;
        if (r >= n) r -= n;
        return static_cast<const T*>(p.grad[base + r]) + sg.off;
    };
    auto out = [&](int o) { return static_cast<T*>(p.grad[base + o]) + sg.off; };
    const uint64_t len = sg.len;
    uint64_t head = (uint64_t)((L - phase_of(in(0), L)) & (L - 1));
    if (head > len) head = len;
    const uint64_t nv = (len - head) / L;
    const uint64_t tail = len - head - nv * L;
    if (tile == 0 && (uint64_t)threadIdx.x < head + tail) {
        const uint64_t e = (uint64_t)threadIdx.x < head ? (uint64_t)threadIdx.x : head + nv * L + (threadIdx.x - head);
        fold_one<G, OP, 0>(in, n, out, n, e, p.divisor);
    }
    const uint64_t v0 = tile * TV;
    if (v0 >= nv) return;
    const uint32_t nvt = (uint32_t)(nv - v0 < TV ? nv - v0 : TV);
    const uint32_t bytes = nvt * 16u;
    const uint64_t e0 = head + v0 * L;  // 16-byte aligned in every rank's copy

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
        G::unpack(sm[v], a);
#pragma unroll 4
        for (int j = 1; j < (NS > 0 ? NS : n); ++j) {
            Acc x[L];
            G::unpack(sm[j * TV + v], x);
#pragma unroll
            for (int l = 0; l < L; ++l) a[l] = apply<OP>(a[l], x[l]);
        }
#pragma unroll
        for (int l = 0; l < L; ++l) a[l] = finish_n<OP, NS>(a[l], p.divisor);
        sm[v] = G::pack(a);  // one rounding to the gradient type, into slot 0
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int o = 0; o < n; ++o)
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
                         ::"l"(out(o) + e0), "r"(bulk_smem_addr(sm)), "r"(bytes)
                         : "memory");
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
        bulk_bar_inval(b);
    }
}

// Elements per bulk tile of the bucket sync: the whole vectors of one rank's
// share of the tile bytes (the compiled counts 2, 4, 8 and 16 tile alike).
uint64_t bucket_bulk_tile_elems(int grad_dtype, int n)
{
    return (uint64_t)bulk_tile_vectors(n) * (grad_dtype == kF32 ? 4u : 8u);
}

template <class G, int OP>
cudaError_t launch_bucket_bulk(const BucketFoldParams& p, int grad_dtype, cudaStream_t s, bool pdl, bool* launched)
{
    *launched = false;
    RankParams rp{};
    rp.waits = bulk_wait_counters();  // once per launch
    if (!rp.waits) return cudaSuccess;
    const BulkParams wait = bulk_params(rp);
    auto* bp = new BucketBulkParams();
    bp->f = p;
    bp->waits = wait.waits;
    bp->hold = wait.hold;
    bp->spin = wait.spin;
    const uint64_t te = bucket_bulk_tile_elems(grad_dtype, p.n);
    bp->f.tile0[0] = 0;
    for (int i = 0; i < p.nseg; ++i)  // every non-empty segment has a tile 0 for its head and tail
        bp->f.tile0[i + 1] = bp->f.tile0[i] + (p.seg[i].len ? (p.seg[i].len + te - 1) / te : 0);
    const uint64_t work = bp->f.tile0[p.nseg];
    cudaError_t e = cudaSuccess;
    if (work > 0 && work <= kMaxGrid) {
        *launched = true;
        bp->tv = bulk_tile_vectors(p.n);
        auto go = [&](void (*kernel)(BucketBulkParams), uint32_t smem) {
            cudaLaunchAttribute attr{};
            attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
            attr.val.programmaticStreamSerializationAllowed = 1;
            cudaLaunchConfig_t cfg{};
            cfg.gridDim = dim3((unsigned)work);
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = smem;
            cfg.stream = s;
            cfg.attrs = &attr;
            cfg.numAttrs = pdl ? 1 : 0;
            return cudaLaunchKernelEx(&cfg, kernel, *bp);
        };
        switch (p.n) {
        case 2: e = go(bucket_bulk_kernel<G, OP, 2>, bulk_smem<2>()); break;
        case 4: e = go(bucket_bulk_kernel<G, OP, 4>, bulk_smem<4>()); break;
        case 8: e = go(bucket_bulk_kernel<G, OP, 8>, bulk_smem<8>()); break;
        case 16: e = go(bucket_bulk_kernel<G, OP, 16>, bulk_smem<16>()); break;
        default: e = go(bucket_bulk_kernel<G, OP, 0>, bp->tv * 16u * (uint32_t)p.n);
        }
        if (e == cudaSuccess) e = cudaGetLastError();
    } else if (work == 0) {
        *launched = true;
    }
    delete bp;
    return e;
}

template <class P>
cudaError_t launch_all_b(void (*kernel)(P), const P& p, uint64_t work, cudaStream_t s, uint64_t max_grid = kMaxGrid)
{
    if (work == 0) return cudaSuccess;
    const uint64_t grid = work < max_grid ? work : max_grid;
    kernel<<<(unsigned)grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <class G, int OP>
cudaError_t launch_fold(const BucketFoldParams& p, uint64_t work, cudaStream_t s, uint64_t max_grid)
{
    constexpr int V = kVptReduce;
    switch (p.n) {
    case 2: return launch_all_b(bucket_fold_kernel<G, OP, V, 1, 2>, p, work, s, max_grid);
    case 4: return launch_all_b(bucket_fold_kernel<G, OP, V, 3, 4>, p, work, s, max_grid);
    case 8: return launch_all_b(bucket_fold_kernel<G, OP, V, 7, 8>, p, work, s, max_grid);
    }
    return launch_all_b(bucket_fold_kernel<G, OP, V, kGroup, 0>, p, work, s, max_grid);
}

}  // namespace

// Elements one pack/unpack tile covers: kThreads * kUnitsPerThread 16-byte
// vectors of the gradient type (8 elements each for bf16 and fp16, 4 for fp32).
uint64_t bucket_tile_elems(int grad_dtype)
{
    return (uint64_t)kThreads * kUnitsPerThread * (grad_dtype == kBF16 || grad_dtype == kF16 ? 8u : 4u);
}

cudaError_t launch_bucket_pack(int grad_dtype, const BucketCopyParams& p, cudaStream_t s)
{
    const uint64_t work = p.tile0[p.nt];
    if (grad_dtype == kBF16) return launch_all_b(bucket_pack_kernel<BF16T>, p, work, s);
    if (grad_dtype == kF16) return launch_all_b(bucket_pack_kernel<F16T>, p, work, s);
    if (grad_dtype == kF32) return launch_all_b(bucket_pack_kernel<F32T>, p, work, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bucket_unpack(int grad_dtype, int op, const BucketCopyParams& p, cudaStream_t s)
{
    const uint64_t work = p.tile0[p.nt];
    const bool avg = op == kAvg;
    if (grad_dtype == kBF16)
        return avg ? launch_all_b(bucket_unpack_kernel<BF16T, kAvg>, p, work, s)
                   : launch_all_b(bucket_unpack_kernel<BF16T, kSum>, p, work, s);
    if (grad_dtype == kF16)
        return avg ? launch_all_b(bucket_unpack_kernel<F16T, kAvg>, p, work, s)
                   : launch_all_b(bucket_unpack_kernel<F16T, kSum>, p, work, s);
    if (grad_dtype == kF32)
        return avg ? launch_all_b(bucket_unpack_kernel<F32T, kAvg>, p, work, s)
                   : launch_all_b(bucket_unpack_kernel<F32T, kSum>, p, work, s);
    return cudaErrorInvalidValue;
}

cudaError_t launch_bucket_fold(int grad_dtype, int op, const BucketFoldParams& p, cudaStream_t s, uint64_t max_grid,
                               bool pdl)
{
    const uint64_t work = p.tile0[p.nseg];
    const bool avg = op == kAvg;
    // the bulk-copy fold when it applies (no CTA cap: one CTA per tile)
    if (max_grid >= kMaxGrid && p.vec_ok && p.n >= 2) {
        bool launched = false;
        cudaError_t e = cudaSuccess;
        if (grad_dtype == kBF16)
            e = avg ? launch_bucket_bulk<BF16T, kAvg>(p, grad_dtype, s, pdl, &launched)
                    : launch_bucket_bulk<BF16T, kSum>(p, grad_dtype, s, pdl, &launched);
        else if (grad_dtype == kF16)
            e = avg ? launch_bucket_bulk<F16T, kAvg>(p, grad_dtype, s, pdl, &launched)
                    : launch_bucket_bulk<F16T, kSum>(p, grad_dtype, s, pdl, &launched);
        else if (grad_dtype == kF32)
            e = avg ? launch_bucket_bulk<F32T, kAvg>(p, grad_dtype, s, pdl, &launched)
                    : launch_bucket_bulk<F32T, kSum>(p, grad_dtype, s, pdl, &launched);
        if (e != cudaSuccess || launched) return e;
    }
    if (grad_dtype == kBF16)
        return avg ? launch_fold<BF16T, kAvg>(p, work, s, max_grid) : launch_fold<BF16T, kSum>(p, work, s, max_grid);
    if (grad_dtype == kF16)
        return avg ? launch_fold<F16T, kAvg>(p, work, s, max_grid) : launch_fold<F16T, kSum>(p, work, s, max_grid);
    if (grad_dtype == kF32)
        return avg ? launch_fold<F32T, kAvg>(p, work, s, max_grid) : launch_fold<F32T, kSum>(p, work, s, max_grid);
    return cudaErrorInvalidValue;
}

}  // namespace rr
