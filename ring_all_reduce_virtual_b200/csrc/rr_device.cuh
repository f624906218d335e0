// rr_device.cuh -- device building blocks shared by the kernels: element
// types, the reduction operators, 128-bit memory access and the tile routine
// that folds (or copies) one tile of one segment.
//
// A "segment" is a run of `len` elements that all reduce in the same order:
// a chunk of the all-reduce (its fold starts on rank c, [P4] "Ring all-reduce
// and communication volume"), one rank's part of a reduce-scatter, one ring
// step's chunk transfer, one tensor of a bucket.  A segment has `nin` input
// pointers in fold order and `nout` output pointers; the fold of element e is
// op(...op(op(in0[e], in1[e]), in2[e])..., in_{nin-1}[e]), then AVG's division
// by the rank count, then a store to every output.
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks);
// [P1] "How all-reduce keeps every card identical" (mhpq.cn), s2.1 for the
// operators and s5.3 for reducing low-precision gradients in fp32.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace rr {

constexpr int kMaxRanks = 64;
constexpr int kThreads = 256;  // threads per CTA of every kernel
constexpr int kGroup = 8;      // input ranks whose loads are issued together (N-input folds)

enum OpCode : int { kSum = 0, kAvg = 1, kMax = 2, kMin = 3, kProd = 4 };

// ------------------------------------------------------------ element types

// fp32 buffers, fp32 arithmetic; 4 elements per 16-byte vector.
struct F32T {
    using T = float;
    using Acc = float;
    static constexpr int L = 4;
    __device__ static __forceinline__ Acc ld1(const T* p) { return *p; }
    __device__ static __forceinline__ void st1(T* p, Acc v) { *p = v; }
    __device__ static __forceinline__ void unpack(const uint4& r, Acc (&a)[L])
    {
        a[0] = __uint_as_float(r.x);
        a[1] = __uint_as_float(r.y);
        a[2] = __uint_as_float(r.z);
        a[3] = __uint_as_float(r.w);
    }
    __device__ static __forceinline__ uint4 pack(const Acc (&a)[L])
    {
        return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                          __float_as_uint(a[3]));
    }
};

// bf16 buffers (raw 16-bit patterns), fp32 arithmetic; widening is the exact
// shift into the top half of a binary32, narrowing rounds to nearest even.
struct BF16T {
    using T = uint16_t;
    using Acc = float;
    static constexpr int L = 8;
    __device__ static __forceinline__ Acc ld1(const T* p) { return __uint_as_float((uint32_t)*p << 16); }
    __device__ static __forceinline__ void st1(T* p, Acc v)
    {
        *p = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    }
    __device__ static __forceinline__ void unpack2(uint32_t w, Acc& lo, Acc& hi)
    {
        lo = __uint_as_float(w << 16);
        hi = __uint_as_float(w & 0xffff0000u);
    }
    __device__ static __forceinline__ uint32_t pack2(Acc lo, Acc hi)
    {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ static __forceinline__ void unpack(const uint4& r, Acc (&a)[L])
    {
        unpack2(r.x, a[0], a[1]);
        unpack2(r.y, a[2], a[3]);
        unpack2(r.z, a[4], a[5]);
        unpack2(r.w, a[6], a[7]);
    }
    __device__ static __forceinline__ uint4 pack(const Acc (&a)[L])
    {
        return make_uint4(pack2(a[0], a[1]), pack2(a[2], a[3]), pack2(a[4], a[5]), pack2(a[6], a[7]));
    }
};

// fp16 buffers (raw IEEE binary16 patterns), fp32 arithmetic; widening is
// exact, narrowing rounds to nearest even (overflow to infinity).
struct F16T {
    using T = uint16_t;
    using Acc = float;
    static constexpr int L = 8;
    __device__ static __forceinline__ Acc ld1(const T* p) { return __half2float(__ushort_as_half(*p)); }
    __device__ static __forceinline__ void st1(T* p, Acc v) { *p = __half_as_ushort(__float2half_rn(v)); }
    __device__ static __forceinline__ void unpack2(uint32_t w, Acc& lo, Acc& hi)
    {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));  // .x = low half
        lo = f.x;
        hi = f.y;
    }
    __device__ static __forceinline__ uint32_t pack2(Acc lo, Acc hi)
    {
        __half2 h = __floats2half2_rn(lo, hi);  // .x = lo (low half), .y = hi
        return *reinterpret_cast<uint32_t*>(&h);
    }
    __device__ static __forceinline__ void unpack(const uint4& r, Acc (&a)[L])
    {
        unpack2(r.x, a[0], a[1]);
        unpack2(r.y, a[2], a[3]);
        unpack2(r.z, a[4], a[5]);
        unpack2(r.w, a[6], a[7]);
    }
    __device__ static __forceinline__ uint4 pack(const Acc (&a)[L])
    {
        return make_uint4(pack2(a[0], a[1]), pack2(a[2], a[3]), pack2(a[4], a[5]), pack2(a[6], a[7]));
    }
};

// int32 buffers; SUM and PROD wrap modulo 2^32.
struct I32T {
    using T = int32_t;
    using Acc = int32_t;
    static constexpr int L = 4;
    __device__ static __forceinline__ Acc ld1(const T* p) { return *p; }
    __device__ static __forceinline__ void st1(T* p, Acc v) { *p = v; }
    __device__ static __forceinline__ void unpack(const uint4& r, Acc (&a)[L])
    {
        a[0] = (int32_t)r.x;
        a[1] = (int32_t)r.y;
        a[2] = (int32_t)r.z;
        a[3] = (int32_t)r.w;
    }
    __device__ static __forceinline__ uint4 pack(const Acc (&a)[L])
    {
        return make_uint4((uint32_t)a[0], (uint32_t)a[1], (uint32_t)a[2], (uint32_t)a[3]);
    }
};

// -------------------------------------------------------------- operators

// One binary step of the fold, partial on the left.  __fadd_rn/__fmul_rn are
// never contracted into an FMA; MAX/MIN keep the left operand on ties.
template <int OP>
__device__ __forceinline__ float apply(float a, float b)
{
    if constexpr (OP == kSum || OP == kAvg) return __fadd_rn(a, b);
    else if constexpr (OP == kProd) return __fmul_rn(a, b);
    else if constexpr (OP == kMax) return (a < b) ? b : a;
    else return (b < a) ? b : a;
}

template <int OP>
__device__ __forceinline__ int32_t apply(int32_t a, int32_t b)
{
    if constexpr (OP == kSum) return (int32_t)((uint32_t)a + (uint32_t)b);
    else if constexpr (OP == kProd) return (int32_t)((uint32_t)a * (uint32_t)b);
    else if constexpr (OP == kMax) return (a < b) ? b : a;
    else return (b < a) ? b : a;
}

// AVG's last step: one IEEE division of the full fold by the rank count.
// When the count is a power of two its reciprocal is exact, and a * (1/N) is
// then the same correctly rounded value of the same real quotient as a / N,
// so the cheaper multiply gives identical bits.
__device__ __forceinline__ bool is_pow2(float d)
{
    const uint32_t u = __float_as_uint(d);
    return (u & 0x007fffffu) == 0u && d >= 1.0f;  // positive, normal, zero mantissa
}

// The exact reciprocal of a power of two 2^k (|k| < 126): the exponent
// negated, no reciprocal instruction.
__device__ __forceinline__ float pow2_reciprocal(float d)
{
    return __uint_as_float(0x7f000000u - (__float_as_uint(d) & 0x7f800000u));
}

// The correctly rounded fp64 reciprocals of the rank counts 1..kMaxRanks,
// evaluated by the compiler (IEEE division in a constant expression).
struct CountReciprocals {
    double v[kMaxRanks + 1];
};
constexpr CountReciprocals count_reciprocals()
{
    CountReciprocals r{};
    for (int i = 1; i <= kMaxRanks; ++i) r.v[i] = 1.0 / (double)i;
    return r;
}
static __constant__ CountReciprocals kCountReciprocals = count_reciprocals();

// Any other whole rank count N (below 2^24) takes no division either: the
// fp64 product of a and the correctly rounded fp64 reciprocal of N, rounded
// once to fp32, is a / N correctly rounded.  The product's relative error is
// below 2^-52; the exact quotient's relative distance to the nearest fp32
// rounding boundary is at least 2^-25 / N, because a boundary m (a midpoint
// between neighbouring fp32 values) is an odd multiple of its binade's step
// 2^(E-24), a (whose binade is not below E) and N * m are multiples of that
// step, and a == N * m is impossible: for N not a power of two, N * m has
// more than 24 significant bits.  So both roundings land on the same side of
// every boundary, for subnormal quotients, zeros and infinities too.  (The
// division sequence this replaces cost up to 20 % of the time of a bucket
// unpack at 3, 5 or 6 ranks, where it runs once per element per rank.)
__device__ __forceinline__ bool is_whole_count(float d)
{
    return d >= 1.0f && d < 16777216.0f && d == truncf(d);
}

template <int OP>
__device__ __forceinline__ float finish(float a, float divisor)
{
    if constexpr (OP == kAvg) {
        if (is_pow2(divisor)) return __fmul_rn(a, pow2_reciprocal(divisor));
        if (is_whole_count(divisor)) {
            const uint32_t k = (uint32_t)divisor;
            const double r = k <= (uint32_t)kMaxRanks ? kCountReciprocals.v[k] : __drcp_rn((double)divisor);
            return __double2float_rn(__dmul_rn((double)a, r));
        }
        return __fdiv_rn(a, divisor);
    } else {
        return a;
    }
}

template <int OP>
__device__ __forceinline__ int32_t finish(int32_t a, float) { return a; }

// finish() for a rank count NS fixed at compile time (0: use the runtime
// divisor): a power-of-two NS multiplies by its exact reciprocal, a constant.
template <int OP, int NS>
__device__ __forceinline__ float finish_n(float a, float divisor)
{
    if constexpr (OP == kAvg && NS > 0 && (NS & (NS - 1)) == 0) return __fmul_rn(a, 1.0f / (float)NS);
    else return finish<OP>(a, divisor);
}

template <int OP, int NS>
__device__ __forceinline__ int32_t finish_n(int32_t a, float) { return a; }

// The bf16 wire format: a value as it arrives after crossing a link that
// carries bf16 (round to nearest even, back to fp32 exactly).
__device__ __forceinline__ float wire_q(float v)
{
    return __uint_as_float((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v)) << 16);
}

// WIRE modes of the folds: 0 exact transfers; 1 the partial is rounded to the
// wire format before each fold step and the result before it is stored (it is
// what the all-gather sends); 2 partials only (a reduce-scatter step that does
// not complete its chunk).
template <int WIRE>
__device__ __forceinline__ float wire_in(float a)
{
    if constexpr (WIRE != 0) return wire_q(a);
    else return a;
}

template <int WIRE>
__device__ __forceinline__ int32_t wire_in(int32_t a) { return a; }

template <int WIRE>
__device__ __forceinline__ float wire_out(float a)
{
    if constexpr (WIRE == 1) return wire_q(a);
    else return a;
}

template <int WIRE>
__device__ __forceinline__ int32_t wire_out(int32_t a) { return a; }

// ------------------------------------------------------------------ memory

// 128-bit streaming access: every byte is touched once per call, so hint the
// caches to evict it first.  Plain (coherent) loads: in-place calls read and
// write the same buffers.
__device__ __forceinline__ uint4 ldv(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }
__device__ __forceinline__ void stv(void* p, const uint4& v) { __stcs(reinterpret_cast<uint4*>(p), v); }

template <class T>
__device__ __forceinline__ int phase_of(const T* p, int L)
{
    return (int)(((uintptr_t)p / sizeof(T)) & (uintptr_t)(L - 1));
}

// Store the elements of one 16-byte vector one by one (at an address that is
// not 16-byte aligned): the bits as they are.
template <class T>
__device__ __forceinline__ void st_lanes(T* q, const uint4& r)
{
    constexpr int L = 16 / (int)sizeof(T);
    const T* e = reinterpret_cast<const T*>(&r);
#pragma unroll
    for (int l = 0; l < L; ++l) q[l] = e[l];
}

// The 16 bytes that start b bytes into the 32-byte window lo:hi (0 < b < 16,
// b even: a whole number of 16- or 32-bit elements).
__device__ __forceinline__ uint4 shift_window(const uint4& lo, const uint4& hi, int b)
{
    uint32_t w0, w1, w2, w3, w4;  // five words from word b / 4 on
    switch (b >> 2) {
    case 0: w0 = lo.x; w1 = lo.y; w2 = lo.z; w3 = lo.w; w4 = hi.x; break;
    case 1: w0 = lo.y; w1 = lo.z; w2 = lo.w; w3 = hi.x; w4 = hi.y; break;
    case 2: w0 = lo.z; w1 = lo.w; w2 = hi.x; w3 = hi.y; w4 = hi.z; break;
    default: w0 = lo.w; w1 = hi.x; w2 = hi.y; w3 = hi.z; w4 = hi.w; break;
    }
    if (b & 3)
        return make_uint4(__funnelshift_r(w0, w1, 16), __funnelshift_r(w1, w2, 16), __funnelshift_r(w2, w3, 16),
                          __funnelshift_r(w3, w4, 16));
    return make_uint4(w0, w1, w2, w3);
}

// --------------------------------------------------------------- the tile

// Scalar fold of element e of a segment.
template <class Ty, int OP, int WIRE, class InF, class OutF>
__device__ __forceinline__ void fold_one(const InF& in, int nin, const OutF& out, int nout, uint64_t e,
                                         float divisor)
{
    using Acc = typename Ty::Acc;
    Acc acc = Ty::ld1(in(0) + e);
    for (int j = 1; j < nin; ++j) acc = apply<OP>(wire_in<WIRE>(acc), Ty::ld1(in(j) + e));
    if (nin > 1) acc = wire_out<WIRE>(finish<OP>(acc, divisor));
    for (int o = 0; o < nout; ++o) Ty::st1(out(o) + e, acc);
}

// Fold (nin > 1) or copy (nin == 1) tile `tile` of a segment of `len`
// elements.  VPT is the number of 16-byte vectors per thread per tile, G the
// number of further input ranks whose loads are issued before they are
// folded: every thread keeps up to VPT * (G + 1) loads in flight.  NS > 0 is
// the rank count (AVG's divisor) when it is fixed at compile time; WIRE
// selects the bf16 wire format (see wire_in / wire_out).  in(j) /
// out(o) return the segment's base pointers.  vec_ok says
// that every in(j) has the same address modulo 16 as in(0), and every out(o)
// the same as out(0) (checked by the host); then the segment splits into a
// scalar head up to the inputs' first 16-byte boundary, a body of 16-byte
// vectors and a scalar tail -- each vector stored whole when out(0) has the
// inputs' phase, element by element otherwise -- and without vec_ok every
// element is scalar.  Tile t covers body vectors [t*TV, (t+1)*TV), TV =
// kThreads*VPT, or the same number of elements on the scalar path; tile 0
// also does the head and tail.
template <class Ty, int OP, int VPT, int G, int NS = 0, int WIRE = 0, class InF, class OutF>
__device__ __forceinline__ void fold_tile(const InF& in, int nin, const OutF& out, int nout, uint64_t len,
                                          uint64_t tile, bool vec_ok, float divisor)
{
    using T = typename Ty::T;
    using Acc = typename Ty::Acc;
    constexpr int L = Ty::L;
    constexpr uint64_t TV = (uint64_t)kThreads * VPT;
    const int tid = threadIdx.x;
    const int pin = phase_of(in(0), L);
    const int pout = phase_of(out(0), L);
    const bool whole = pin == pout;  // results stored as whole vectors
    if (!vec_ok) {
        const uint64_t e0 = tile * TV * L;
#pragma unroll 4
        for (int k = 0; k < VPT * L; ++k) {
            uint64_t e = e0 + (uint64_t)k * kThreads + tid;
            if (e < len) fold_one<Ty, OP, WIRE>(in, nin, out, nout, e, divisor);
        }
        return;
    }
    uint64_t head = (uint64_t)((L - pin) & (L - 1));
    if (head > len) head = len;
    const uint64_t nv = (len - head) / L;
    const uint64_t tail = len - head - nv * L;
    if (tile == 0 && (uint64_t)tid < head + tail) {
        uint64_t e = (uint64_t)tid < head ? (uint64_t)tid : head + nv * L + ((uint64_t)tid - head);
        fold_one<Ty, OP, WIRE>(in, nin, out, nout, e, divisor);
    }
    const uint64_t v0 = tile * TV;
    if (v0 >= nv) return;
    uint64_t off[VPT];
    bool ok[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
        uint64_t v = v0 + (uint64_t)u * kThreads + tid;
        ok[u] = v < nv;
        off[u] = head + v * L;
    }
    if (nin == 1) {  // a copy: move the raw bits
        uint4 raw[VPT];
        const T* p = in(0);
#pragma unroll
        for (int u = 0; u < VPT; ++u)
            if (ok[u]) raw[u] = ldv(p + off[u]);
#pragma unroll 4
        for (int o = 0; o < nout; ++o) {
            T* q = out(o);
#pragma unroll
            for (int u = 0; u < VPT; ++u)
                if (ok[u]) {
                    if (whole) stv(q + off[u], raw[u]);
                    else st_lanes(q + off[u], raw[u]);
                }
        }
        return;
    }
    Acc a[VPT][L];
    {
        const T* p = in(0);
#pragma unroll
        for (int u = 0; u < VPT; ++u)
            if (ok[u]) Ty::unpack(ldv(p + off[u]), a[u]);
    }
    for (int g = 1; g < nin; g += G) {
        uint4 raw[G][VPT];
#pragma unroll
        for (int k = 0; k < G; ++k) {
            if (g + k < nin) {
                const T* p = in(g + k);
#pragma unroll
                for (int u = 0; u < VPT; ++u)
                    if (ok[u]) raw[k][u] = ldv(p + off[u]);
            }
        }
#pragma unroll
        for (int k = 0; k < G; ++k) {
            if (g + k < nin) {
#pragma unroll
                for (int u = 0; u < VPT; ++u) {
                    Acc b[L];
                    Ty::unpack(raw[k][u], b);
#pragma unroll
                    for (int l = 0; l < L; ++l) a[u][l] = apply<OP>(wire_in<WIRE>(a[u][l]), b[l]);
                }
            }
        }
    }
    uint4 res[VPT];
#pragma unroll
    for (int u = 0; u < VPT; ++u) {
#pragma unroll
        for (int l = 0; l < L; ++l) a[u][l] = wire_out<WIRE>(finish_n<OP, NS>(a[u][l], divisor));
        res[u] = Ty::pack(a[u]);
    }
#pragma unroll 4
    for (int o = 0; o < nout; ++o) {
        T* q = out(o);
#pragma unroll
        for (int u = 0; u < VPT; ++u)
            if (ok[u]) {
                if (whole) stv(q + off[u], res[u]);
                else st_lanes(q + off[u], res[u]);
            }
    }
}

}  // namespace rr
