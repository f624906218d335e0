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
#include "rr_device.cuh"
#include "rr_internal.h"

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
};

template <>
struct Quad<BF16T> : Quad16<BF16T> {};

template <>
struct Quad<F16T> : Quad16<F16T> {};

// Convert one tile of a segment from In's element type to Out's, dividing by
// `divisor` first when OP is AVG.  A tile is kThreads * Q quads, Q chosen so
// that it covers kThreads * kUnitsPerThread 16-byte vectors of the narrower
// type (bucket_tile_elems).  When src and dst reach a quad boundary after the
// same scalar head, the body moves quads and tile 0 also does the head and
// the tail (< 4 elements each); otherwise every element is scalar.
template <class In, class Out, int OP, int Q = kUnitsPerThread * (In::L > Out::L ? In::L : Out::L) / 4>
__device__ __forceinline__ void convert_tile(const typename In::T* src, typename Out::T* dst, uint64_t len,
                                             uint64_t tile, bool vec_ok, float divisor)
{
    constexpr uint64_t TQ = (uint64_t)kThreads * Q;  // Q: quads per thread per tile
    const int tid = threadIdx.x;
    const int ps = phase_of(src, 4), pd = phase_of(dst, 4);
    auto one = [&](uint64_t e) { Out::st1(dst + e, finish<OP>((float)In::ld1(src + e), divisor)); };
    if (!(vec_ok && ps == pd)) {
        const uint64_t e0 = tile * TQ * 4;
#pragma unroll 4
        for (int k = 0; k < Q * 4; ++k) {
            const uint64_t e = e0 + (uint64_t)k * kThreads + tid;
            if (e < len) one(e);
        }
        return;
    }
    uint64_t head = (uint64_t)((4 - ps) & 3);
    if (head > len) head = len;
    const uint64_t nq = (len - head) / 4;
    const uint64_t tail = len - head - nq * 4;
    if (tile == 0 && (uint64_t)tid < head + tail)
        one((uint64_t)tid < head ? (uint64_t)tid : head + nq * 4 + ((uint64_t)tid - head));
    // all of this thread's loads first (Q in flight), then the conversions
    // and stores
    typename Quad<In>::R raw[Q];
    uint64_t e[Q];
    bool ok[Q];
#pragma unroll
    for (int k = 0; k < Q; ++k) {
        const uint64_t q = tile * TQ + (uint64_t)k * kThreads + tid;
        ok[k] = q < nq;
        e[k] = head + q * 4;
        if (ok[k]) raw[k] = Quad<In>::ld(src + e[k]);
    }
#pragma unroll
    for (int k = 0; k < Q; ++k) {
        if (!ok[k]) continue;
        float a[4];
        Quad<In>::to_f(raw[k], a);
#pragma unroll
        for (int l = 0; l < 4; ++l) a[l] = finish<OP>(a[l], divisor);
        Quad<Out>::st(dst + e[k], Quad<Out>::from_f(a));
    }
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
        convert_tile<G, F32T, kSum>(src, dst, p.tlen[t], tile, p.vec_ok, 1.0f);
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
        convert_tile<F32T, G, OP>(src, dst, p.tlen[t], tile, p.vec_ok, p.divisor);
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

cudaError_t launch_bucket_fold(int grad_dtype, int op, const BucketFoldParams& p, cudaStream_t s, uint64_t max_grid)
{
    const uint64_t work = p.tile0[p.nseg];
    const bool avg = op == kAvg;
    if (grad_dtype == kBF16)
        return avg ? launch_fold<BF16T, kAvg>(p, work, s, max_grid) : launch_fold<BF16T, kSum>(p, work, s, max_grid);
    if (grad_dtype == kF16)
        return avg ? launch_fold<F16T, kAvg>(p, work, s, max_grid) : launch_fold<F16T, kSum>(p, work, s, max_grid);
    if (grad_dtype == kF32)
        return avg ? launch_fold<F32T, kAvg>(p, work, s, max_grid) : launch_fold<F32T, kSum>(p, work, s, max_grid);
    return cudaErrorInvalidValue;
}

}  // namespace rr
