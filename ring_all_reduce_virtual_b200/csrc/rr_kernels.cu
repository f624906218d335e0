// rr_kernels.cu -- the collectives' kernels and their launchers.
//
// All kernels are HBM-bound streaming kernels: each input byte is read once
// and each output byte written once per launch (a source tile that several
// outputs need is read from L2 after the first), with 128-bit vector access
// and one CTA per (segment, tile) work item (a grid-stride loop covers grids
// past the launch limit).  No kernel waits on another CTA or another launch.
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "The five primitives", "Ring all-reduce and communication volume"
// and "alpha-beta model"; [P3] "Training gradient sync and collective
// communication" (geek-doc.cn), sections 3 and 6.
#include "rr_launch.cuh"
#include "rr_oneshot.cuh"

namespace rr {

namespace {


// Copy tile `tile` of a segment of `len` elements, in -> out, the bits as
// they are; tiles as fold_tile's with VPT vectors per thread.  When in and
// out have the same 16-byte phase: whole vectors (fold_tile's copy path).
// Otherwise the tile's vectors are aligned to the output, and their source
// elements, d = (phase of in - phase of out) mod L elements into an aligned
// input vector, are copied aligned -- one asynchronous copy per input vector,
// plus the one after, which holds the last few elements -- into shared
// memory; each
// output vector reads the two stage vectors it straddles and shifts them in
// registers, so every access is a whole aligned vector and no global load is
// issued twice.  Every thread of the CTA calls this for the same tile.
template <class Ty, int VPT>
__device__ __forceinline__ void copy_tile(const typename Ty::T* in, typename Ty::T* out, uint64_t len, uint64_t tile)
{
    using T = typename Ty::T;
    constexpr int L = Ty::L;
    constexpr uint32_t TV = (uint32_t)kThreads * VPT;
    const int pin = phase_of(in, L), pout = phase_of(out, L);
    if (pin == pout) {
        auto i0 = [&](int) { return in; };
        auto o0 = [&](int) { return out; };
        fold_tile<Ty, kSum, VPT, 1>(i0, 1, o0, 1, len, tile, true, 1.0f);
        return;
    }
    uint64_t head = (uint64_t)((L - pout) & (L - 1));
    if (head > len) head = len;
    const uint64_t nv = (len - head) / L, tail = len - head - nv * L;
    if (tile == 0 && (uint64_t)threadIdx.x < head + tail) {
        const uint64_t e = (uint64_t)threadIdx.x < head ? (uint64_t)threadIdx.x : head + nv * L + (threadIdx.x - head);
        out[e] = in[e];
    }
    const uint64_t v0 = tile * TV;
    if (v0 >= nv) return;
    const uint32_t nvt = nv - v0 < TV ? (uint32_t)(nv - v0) : TV;
    const int d = (pin - pout) & (L - 1);
    const T* ib = reinterpret_cast<const T*>(reinterpret_cast<uintptr_t>(in + head + v0 * L) - (uintptr_t)d * sizeof(T));
    __shared__ __align__(16) uint4 stage[TV + 1];
    // global -> shared without passing through registers (the one-to-many
    // copies run at 32 registers a thread), all of the thread's copies in flight
#pragma unroll
    for (int k = 0; k <= VPT; ++k) {
        const uint32_t i = (uint32_t)k * kThreads + threadIdx.x;
        if (i <= nvt)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(&stage[i])),
                         "l"(ib + (uint64_t)i * L)
                         : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
#pragma unroll 1
    for (int k = 0; k < VPT; ++k) {
        const uint32_t i = (uint32_t)k * kThreads + threadIdx.x;
        if (i >= nvt) continue;
        // two aligned 16-byte reads of the stage, shifted in registers
        stv(out + head + (v0 + i) * L, shift_window(stage[i], stage[i + 1], d * (int)sizeof(T)));
    }
    __syncthreads();  // the stage is free for the CTA's next tile
}

// Copy tile `tile` of `in` to nout outputs out(0..nout-1), all at one 16-byte
// phase: the tile is staged in shared memory once (cp.async, whole aligned
// vectors) and each vector, shifted to the outputs' phase, is stored to every
// output.  Every thread of the CTA calls this for the same tile.
template <class Ty, int VPT, class Out>
__device__ __forceinline__ void fan_tile(const typename Ty::T* in, Out out, int nout, uint64_t len, uint64_t tile)
{
    using T = typename Ty::T;
    constexpr int L = Ty::L;
    constexpr uint32_t TV = (uint32_t)kThreads * VPT;
    const int pout = phase_of(out(0), L);
    const int pin = phase_of(in, L);
    uint64_t head = (uint64_t)((L - pout) & (L - 1));
    if (head > len) head = len;
    const uint64_t nv = (len - head) / L, tail = len - head - nv * L;
    if (tile == 0 && (uint64_t)threadIdx.x < head + tail) {
        const uint64_t e = (uint64_t)threadIdx.x < head ? (uint64_t)threadIdx.x : head + nv * L + (threadIdx.x - head);
        const T x = in[e];
        for (int j = 0; j < nout; ++j) out(j)[e] = x;
    }
    const uint64_t v0 = tile * TV;
    if (v0 >= nv) return;
    const uint32_t nvt = nv - v0 < TV ? (uint32_t)(nv - v0) : TV;
    const int d = (pin - pout) & (L - 1);
    // d == 0: the tile's own vectors; otherwise one more, for the last shift
    const uint32_t nst = d ? nvt + 1 : nvt;
    const T* ib = reinterpret_cast<const T*>(reinterpret_cast<uintptr_t>(in + head + v0 * L) - (uintptr_t)d * sizeof(T));
    __shared__ __align__(16) uint4 stage[TV + 1];
#pragma unroll
    for (int k = 0; k <= VPT; ++k) {
        const uint32_t i = (uint32_t)k * kThreads + threadIdx.x;
        if (i < nst)
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(&stage[i])),
                         "l"(ib + (uint64_t)i * L)
                         : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
#pragma unroll 1
    for (int k = 0; k < VPT; ++k) {
        const uint32_t i = (uint32_t)k * kThreads + threadIdx.x;
        if (i >= nvt) continue;
        const uint4 v = d ? shift_window(stage[i], stage[i + 1], d * (int)sizeof(T)) : stage[i];
        const uint64_t e = head + (v0 + i) * L;
        for (int j = 0; j < nout; ++j) stv(out(j) + e, v);
    }
    __syncthreads();  // the stage is free for the CTA's next tile
}

// Outputs written per work item by the fan-out forms of the one-to-many
// copies (all-gather, the two-shot's broadcast).  Measured on 2-48 ranks x
// 256 MiB fp32 outputs, whole-vector and odd-sized parts: the all-gather at
// 1 / 2 / 4 / 8 outputs per item ran at 0.87-0.99 / 0.98-1.00 / 0.93-0.98 /
// 0.89-0.98 of the copy peak (one output per item fell off with the rank
// count on odd parts: each item stages and shifts its tile for 16 KB of
// output); the two-shot moved by at most 2 % between 1 and 2.
#ifndef RR_FAN
#define RR_FAN 2
#endif
constexpr int kFan = RR_FAN;

// The one-to-many copies below give each CTA one tile of one or kFan
// outputs (16 KB in, 16 or 32 KB out): such short-lived CTAs keep enough bytes in flight only at
// full occupancy, so they are held to the registers of 8 CTAs per SM
// (measured on the 64-rank all-gather: 6 CTAs per SM ran at 0.86 of the copy
// peak, 8 at 1.03).  The all-to-all reads a separate tile per CTA and ran
// slightly slower with the cap, so it keeps its registers.
constexpr int kSmallCtasPerSm = 8;

// ------------------------------------------------- chunk broadcast
// Two-shot's second shot: segment c = chunk c, read from its owner (rank c)
// and written to chunk c of the N-1 other ranks.  One output per work item
// (ranks at different 16-byte phases):
// item w = (c * tps + tile) * (N-1) + k writes rank k (k < c) or k+1, so the
// N-1 CTAs of a tile run side by side and all but the first read the owner's
// tile from L2 (HBM reads it once).
template <class Ty>
__global__ void __launch_bounds__(kThreads, kSmallCtasPerSm) chunk_bcast_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t m = (uint64_t)p.n - 1;
    const uint64_t total = p.nseg * p.tps * m;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t st = w / m, k = w - st * m;
        const uint64_t c = st / p.tps, tile = st - c * p.tps;
        const uint64_t lo = c * p.C;
        if (lo >= p.count) continue;
        const uint64_t len = p.count - lo < p.C ? p.count - lo : p.C;
        const int owner = (int)c;
        const int dst = (int)k < owner ? (int)k : (int)k + 1;
        copy_tile<Ty, kVptMove>(static_cast<const T*>(p.in[owner]) + lo, static_cast<T*>(p.out[dst]) + lo, len, tile);
    }
}

// The same copies with kFan outputs per work item, when every rank's buffer
// sits at one 16-byte phase: item w = (c * tps + tile) * G + g writes ranks
// g*kFan ... of the N-1 others (G groups), the owner's tile read once per item.
template <class Ty>
__global__ void __launch_bounds__(kThreads, kSmallCtasPerSm) chunk_bcast_fan_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t m = (uint64_t)p.n - 1, ng = (m + kFan - 1) / kFan;
    const uint64_t total = p.nseg * p.tps * ng;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t st = w / ng, g = w - st * ng;
        const uint64_t c = st / p.tps, tile = st - c * p.tps;
        const uint64_t lo = c * p.C;
        if (lo >= p.count) continue;
        const uint64_t len = p.count - lo < p.C ? p.count - lo : p.C;
        const int owner = (int)c, k0 = (int)g * kFan;
        const int nout = (int)m - k0 < kFan ? (int)m - k0 : kFan;
        auto out = [&](int j) {
            const int k = k0 + j;
            return static_cast<T*>(p.out[k < owner ? k : k + 1]) + lo;
        };
        fan_tile<Ty, kVptMove>(static_cast<const T*>(p.in[owner]) + lo, out, nout, len, tile);
    }
}

// -------------------------------------------------- reduce-scatter
// Segment r = part r: fold of in_{r}, in_{r+1}, ... (ring order of chunk r)
// at offset r*C, written to out_r.
template <class Ty, int OP, int VPT, int G, int NS>
__global__ void __launch_bounds__(kThreads) reduce_scatter_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const int n = NS > 0 ? NS : p.n;
    const uint64_t total = p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t r = w / p.tps, tile = w - r * p.tps;
        const uint64_t lo = r * p.C;
        const int start = (int)r;
        auto in = [&](int j) {
            int q = start + j;
            if (q >= n) q -= n;
            return static_cast<const T*>(p.in[q]) + lo;
        };
        auto out = [&](int) { return static_cast<T*>(p.out[start]); };
        fold_tile<Ty, OP, VPT, G, NS>(in, n, out, 1, p.C, tile, p.vec_ok, p.divisor);
    }
}

// ------------------------------------------------------ all-gather
// Segment q = rank q's part, written to offset q*C of every output.  One
// output per work item (outputs at different 16-byte phases): item
// w = (q * tps + tile) * N + o, so the N CTAs of a tile run side by side and
// HBM reads the source tile once (the others hit L2).  Writing all N outputs
// from one CTA measured 0.94 of the copy peak at 8 ranks x 256 MiB.
template <class Ty>
__global__ void __launch_bounds__(kThreads, kSmallCtasPerSm) all_gather_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t n = (uint64_t)p.n;
    const uint64_t total = p.nseg * p.tps * n;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t st = w / n, o = w - st * n;
        const uint64_t q = st / p.tps, tile = st - q * p.tps;
        copy_tile<Ty, kVptMove>(static_cast<const T*>(p.in[q]), static_cast<T*>(p.out[o]) + q * p.C, p.C, tile);
    }
}

// The same copies with kFan outputs per work item, when every output sits at
// one 16-byte phase: item w = (q * tps + tile) * G + g writes outputs
// g*kFan ... (G groups), the source tile read once per item.
template <class Ty>
__global__ void __launch_bounds__(kThreads, kSmallCtasPerSm) all_gather_fan_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t n = (uint64_t)p.n, ng = (n + kFan - 1) / kFan;
    const uint64_t total = p.nseg * p.tps * ng;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t st = w / ng, g = w - st * ng;
        const uint64_t q = st / p.tps, tile = st - q * p.tps;
        const int o0 = (int)g * kFan, nout = (int)n - o0 < kFan ? (int)n - o0 : kFan;
        auto out = [&](int j) { return static_cast<T*>(p.out[o0 + j]) + q * p.C; };
        fan_tile<Ty, kVptMove>(static_cast<const T*>(p.in[q]), out, nout, p.C, tile);
    }
}

// ------------------------------------------------------ all-to-all
// Segment (r, q): block r of rank q goes to block q of rank r.
template <class Ty>
__global__ void __launch_bounds__(kThreads) all_to_all_kernel(const __grid_constant__ RankParams p)
{
    using T = typename Ty::T;
    const uint64_t total = p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t s = w / p.tps, tile = w - s * p.tps;
        const uint64_t r = s / (uint64_t)p.n, q = s - r * (uint64_t)p.n;
        copy_tile<Ty, kVptMove>(static_cast<const T*>(p.in[q]) + r * p.C, static_cast<T*>(p.out[r]) + q * p.C, p.C, tile);
    }
}

// ------------------------------------------------------- table steps
// One ring step or one tree level: every segment folds in0 op in1 into out
// (nin == 2) or copies in0 to out (nin == 1).
// NIN: 2 folds (a reduce-scatter step or reduce level), 1 copies (an
// all-gather step or broadcast level); fixed at compile time.
template <class Ty, int OP, int NIN, int WIRE = 0>
__global__ void __launch_bounds__(kThreads) step_kernel(const __grid_constant__ StepParams p)
{
    using T = typename Ty::T;
    const uint64_t total = (uint64_t)p.nseg * p.tps;
    for (uint64_t w = blockIdx.x; w < total; w += gridDim.x) {
        const uint64_t s = w / p.tps, tile = w - s * p.tps;
        const StepSeg& sg = p.seg[s];
        if (sg.len == 0) continue;
        auto in = [&](int j) { return static_cast<const T*>(j == 0 ? sg.in0 : sg.in1); };
        auto out = [&](int) { return static_cast<T*>(sg.out); };
        fold_tile<Ty, OP, kVptMove, 1, 0, WIRE>(in, NIN, out, 1, sg.len, tile, p.vec_ok, p.divisor);
    }
}

// ------------------------------------------------------------ launching

}  // namespace

uint64_t tile_elems(int dtype, int vpt)
{
    return (uint64_t)kThreads * (uint64_t)vpt * (dtype == kBF16 || dtype == kF16 ? 8u : 4u);
}

namespace {
bool outs_same_phase(const RankParams& p)
{
    for (int r = 1; r < p.n; ++r)
        if ((uintptr_t)p.out[r] % 16 != (uintptr_t)p.out[0] % 16) return false;
    return true;
}
}  // namespace

cudaError_t launch_rank_kernel(int kind, int dtype, int op, const RankParams& p, cudaStream_t s)
{
    uint64_t work = kind == kOneshotTree ? p.tps : p.nseg * p.tps;
    // one output per work item, or kFan when the outputs share a 16-byte phase
    const bool fan = kFan > 1 && outs_same_phase(p);
    const uint64_t per = fan ? (uint64_t)kFan : 1;
    if (kind == kAllGather) work *= ((uint64_t)p.n + per - 1) / per;
    if (kind == kChunkBroadcast) work *= ((uint64_t)p.n - 1 + per - 1) / per;
    if (kind == kAllGather || kind == kAllToAll || kind == kChunkBroadcast) op = kSum;
    const int n = p.n;
    constexpr int V = kVptReduce;
    return with_type(dtype, op, [&]<class Ty, int OP>() -> cudaError_t {
        switch (kind) {
        case kOneshotRing: return launch_oneshot_ring<Ty, OP>(p, work, s);
        case kReduceScatter:
            if (bulk_scatter_eligible(p, (int)sizeof(typename Ty::T))) return launch_scatter_bulk<Ty, OP>(p, s);
            if (!p.vec_ok && mixed_eligible(p, (int)sizeof(typename Ty::T))) return launch_scatter_mixed<Ty, OP>(p, s);
            switch (n) {
            case 2: return launch_all(reduce_scatter_kernel<Ty, OP, V, 1, 2>, p, work, s);
            case 4: return launch_all(reduce_scatter_kernel<Ty, OP, V, 3, 4>, p, work, s);
            case 8: return launch_all(reduce_scatter_kernel<Ty, OP, V, 7, 8>, p, work, s);
            }
            return launch_all(reduce_scatter_kernel<Ty, OP, V, kGroup, 0>, p, work, s);
        case kOneshotTree: return launch_oneshot_tree<Ty, OP>(p, work, s);
        case kAllGather:
            return launch_all(fan ? all_gather_fan_kernel<Ty> : all_gather_kernel<Ty>, p, work, s);
        case kAllToAll: return launch_all(all_to_all_kernel<Ty>, p, work, s);
        case kChunkBroadcast:
            return launch_all(fan ? chunk_bcast_fan_kernel<Ty> : chunk_bcast_kernel<Ty>, p, work, s);
        }
        return cudaErrorInvalidValue;
    });
}

cudaError_t launch_step_wire(int op, int wire, const StepParams& p, cudaStream_t s)
{
    const uint64_t work = (uint64_t)p.nseg * p.tps;
    if (wire == 1)
        return op == kAvg ? launch_all(step_kernel<F32T, kAvg, 2, 1>, p, work, s)
                          : launch_all(step_kernel<F32T, kSum, 2, 1>, p, work, s);
    return op == kAvg ? launch_all(step_kernel<F32T, kAvg, 2, 2>, p, work, s)
                      : launch_all(step_kernel<F32T, kSum, 2, 2>, p, work, s);
}

cudaError_t launch_step(int dtype, int op, const StepParams& p, cudaStream_t s)
{
    const uint64_t work = (uint64_t)p.nseg * p.tps;
    if (p.nin == 1) op = kSum;
    return with_type(dtype, op, [&]<class Ty, int OP>() {
        return p.nin == 2 ? launch_all(step_kernel<Ty, OP, 2>, p, work, s)
                          : launch_all(step_kernel<Ty, kSum, 1>, p, work, s);
    });
}

}  // namespace rr
