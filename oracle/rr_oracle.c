/*
 * rr_oracle.c -- plain, slow, single-purpose CPU oracle for the ring
 * all-reduce over N "virtual ranks" and its companion collectives.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  The product
 * (the CUDA library and its Python binding) never links, loads or calls it,
 * and this file shares no header, helper, table or constant with it.
 *
 * Every rank is one host array.  "Sending" a chunk means copying it into a
 * message buffer; "receiving" means reading the left neighbour's message.
 *
 * Sources (four web pages on ring all-reduce), cited by tag:
 *   [P1] "How all-reduce keeps every card identical" (mhpq.cn, news 451051)
 *   [P2] "AllReduce from principle to tuning" (xxqk.cn, news 376101)
 *   [P3] "Training gradient sync and collective communication: from parameter
 *        server to Ring AllReduce" (geek-doc.cn, training-collective-communication)
 *   [P4] "Collective communication primitives" (ai-infra-handbooks,
 *        train/basics/collectives)
 *
 * Arithmetic precision.  The pages fix the reduction precision for
 * low-precision gradients as fp32 ([P1] s5.3); fp32 buffers are reduced in
 * fp32.  So every floating-point fold here is an fp32 fold, evaluated one
 * IEEE binary32 operation at a time (FLT_EVAL_METHOD == 0, no contraction, no
 * fast-math).  bf16 and fp16 values are carried as their 16-bit patterns.
 *
 * Readings where the pages are silent (stated once, used everywhere):
 *   - chunk size C = ceil(count / N); chunk k is [k*C, min((k+1)*C, count)),
 *     possibly short or empty ([P4] "Ring all-reduce and communication
 *     volume", ring_allreduce.py splits with tensor.chunk(n)).
 *   - the fold of one element is "acc = op(acc, next)": the partial that
 *     arrives first is the left operand.
 *   - max(a, b) = (a < b) ? b : a and min(a, b) = (b < a) ? b : a, so on ties
 *     (including +0 / -0) the left operand is kept.
 *   - AVG = the full fold, then one IEEE division by N ([P1] s2.1 "add, then
 *     divide by N"; [P3] section 3 "sum, then divide by 4").
 *   - bf16 (and fp16) buffers moved by the ring or tree schedules are rounded
 *     back to their type (round to nearest, ties to even) after every hop;
 *     the one-shot definitions fold the widened values in fp32 and round once
 *     at the end.
 *   - int32 SUM and PROD wrap modulo 2^32; AVG is not defined for int32.
 */
#include <float.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#if !defined(FLT_EVAL_METHOD) || FLT_EVAL_METHOD != 0
#error "the oracle needs single-precision evaluation of float expressions"
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_I32 = 2, ORC_F16 = 3 };
enum { ORC_SUM = 0, ORC_AVG = 1, ORC_MAX = 2, ORC_MIN = 3, ORC_PROD = 4 };
enum { ORC_PHASE_RS = 0, ORC_PHASE_AG = 1 };
enum { ORC_OK = 0, ORC_EINVAL = 1, ORC_ENOMEM = 2 };

#ifdef ORC_MUTANTS
/* Planted mistakes, compiled only into the separate mutant build that the
 * test suite uses to show that its pins catch them.  0 = none. */
static int g_mutant = 0;
void orc_set_mutant(int m) { g_mutant = m; }
#define MUTANT(k) (g_mutant == (k))
#else
#define MUTANT(k) 0
#endif

/* One "sent" record of the ring schedule. */
typedef struct {
    int32_t phase;    /* ORC_PHASE_RS or ORC_PHASE_AG */
    int32_t step;     /* 0 .. N-2 within the phase */
    int32_t rank;     /* the sender */
    int32_t dst;      /* the receiver: the right neighbour */
    int32_t send_idx; /* chunk the sender sends */
    int32_t recv_idx; /* chunk the sender receives from its left neighbour */
    uint64_t bytes;   /* bytes of the sent chunk */
} orc_event_t;

/* ---------------------------------------------------------------- bf16 -- */

/* bf16 is the upper half of an IEEE binary32 pattern: widening is exact. */
float orc_bf16_to_f32(uint16_t h)
{
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Narrow binary32 -> bf16 by IEEE round-to-nearest, ties-to-even: drop the
 * low 16 bits, and step the kept part up by one unit when the dropped part is
 * more than half a unit, or exactly half and the kept part is odd.  A carry
 * out of the significand moves into the exponent, which also turns the
 * largest finite values into infinity exactly when IEEE says so.  NaN keeps
 * its sign and becomes a quiet NaN. */
uint16_t orc_f32_to_bf16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu) != 0u)
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t kept = u >> 16;
    uint32_t dropped = u & 0xffffu;
    if (dropped > 0x8000u || (dropped == 0x8000u && (kept & 1u)))
        kept += 1u;
    return (uint16_t)kept;
}

void orc_f32_to_bf16_array(const float* in, uint16_t* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(in[i]);
}

void orc_bf16_to_f32_array(const uint16_t* in, float* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = orc_bf16_to_f32(in[i]);
}

/* ---------------------------------------------------------------- fp16 -- */

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction
 * bits.  Exponent field 0 holds zeros and subnormals (fraction * 2^-24), 31
 * holds infinities and NaNs; every other field e is a normal number
 * (1 + fraction / 2^10) * 2^(e - 15).  Every binary16 value is a binary32
 * value, so widening is exact. */
float orc_f16_to_f32(uint16_t h)
{
    const uint32_t sign = (uint32_t)(h >> 15) << 31;
    const uint32_t e = (h >> 10) & 0x1fu, m = h & 0x3ffu;
    uint32_t u;
    if (e == 0) {  /* zero or subnormal: m * 2^-24, exact in binary32 */
        float f = (float)m * 5.9604644775390625e-08f;
        memcpy(&u, &f, sizeof u);
        u |= sign;
    } else if (e == 31) {
        u = sign | 0x7f800000u | (m << 13) | (m ? 0x00400000u : 0u);  /* inf, or a quiet NaN */
    } else {
        u = sign | ((e - 15u + 127u) << 23) | (m << 13);
    }
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round n / 2^shift to the nearest integer, ties to even (shift >= 1). */
static uint32_t rne_shift(uint32_t n, int shift)
{
    if (shift > 31) return 0;
    const uint32_t q = n >> shift, rem = n & ((1u << shift) - 1u), half = 1u << (shift - 1);
    if (rem > half || (rem == half && (MUTANT(12) || (q & 1u)))) return q + 1u;
    return q;
}

/* Narrow binary32 -> binary16 by round-to-nearest, ties-to-even.  A normal
 * binary32 with unbiased exponent E >= -14 keeps the top 10 of its 23
 * fraction bits, rounded on the 13 dropped ones; a carry out of the fraction
 * moves into the exponent, and exponents past 15 (or a carry into 16) give
 * infinity.  Below 2^-14 the result is the subnormal round(|f| / 2^-24);
 * 1024 there is the smallest normal, 0x0400.  NaN stays a quiet NaN with its
 * sign. */
uint16_t orc_f32_to_f16(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    const uint32_t e32 = (u >> 23) & 0xffu, m32 = u & 0x7fffffu;
    if (e32 == 0xffu) return (uint16_t)(sign | 0x7c00u | (m32 ? 0x0200u | (m32 >> 13) : 0u));
    if (e32 == 0) return sign;  /* binary32 zero or subnormal: below half of 2^-24 */
    const int E = (int)e32 - 127;
    if (E > 15) return (uint16_t)(sign | 0x7c00u);
    const uint32_t sig = m32 | 0x800000u;  /* 24-bit significand: |f| = sig * 2^(E - 23) */
    if (E < -14)                           /* subnormal result: sig * 2^(E - 23) / 2^-24 */
        return (uint16_t)(sign | rne_shift(sig, -1 - E));
    uint32_t bits = ((uint32_t)(E + 15) << 10) + rne_shift(sig, 13) - 0x400u;  /* drop the hidden bit */
    if (bits >= 0x7c00u) bits = 0x7c00u;
    return (uint16_t)(sign | bits);
}

void orc_f32_to_f16_array(const float* in, uint16_t* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = orc_f32_to_f16(in[i]);
}

void orc_f16_to_f32_array(const uint16_t* in, float* out, size_t n)
{
    for (size_t i = 0; i < n; ++i) out[i] = orc_f16_to_f32(in[i]);
}

/* ------------------------------------------------------------- helpers -- */

static size_t esize(int dtype) { return dtype == ORC_BF16 || dtype == ORC_F16 ? 2u : 4u; }

static int valid(int n, int dtype, int op)
{
    if (n < 1) return 0;
    if (dtype != ORC_F32 && dtype != ORC_BF16 && dtype != ORC_I32 && dtype != ORC_F16) return 0;
    if (op < ORC_SUM || op > ORC_PROD) return 0;
    if (dtype == ORC_I32 && op == ORC_AVG) return 0;
    return 1;
}

static int mod(int a, int n) { return ((a % n) + n) % n; }

/* Chunk size C = ceil(count / N). */
size_t orc_chunk_size(size_t count, int n) { return (count + (size_t)n - 1) / (size_t)n; }

/* Number of elements in chunk k (0 for chunks past the end). */
size_t orc_chunk_len(size_t count, int n, int k)
{
    size_t c = orc_chunk_size(count, n);
    size_t lo = (size_t)k * c;
    if (lo >= count) return 0;
    size_t hi = lo + c;
    return (hi > count ? count : hi) - lo;
}

/* The binary operators of [P1] s2.1 (SUM, AVG, MAX, MIN, PROD) on fp32. */
static float op_f32(int op, float a, float b)
{
    switch (op) {
    case ORC_SUM:
    case ORC_AVG:
        return MUTANT(1) ? a - b : a + b;
    case ORC_PROD: return a * b;
    case ORC_MAX: return (a < b) ? b : a;
    case ORC_MIN: return (b < a) ? b : a;
    }
    return a;
}

/* The same operators on int32 (two's complement, SUM and PROD wrap). */
static int32_t op_i32(int op, int32_t a, int32_t b)
{
    switch (op) {
    case ORC_SUM: return (int32_t)((uint32_t)a + (uint32_t)b);
    case ORC_PROD: return (int32_t)((uint32_t)a * (uint32_t)b);
    case ORC_MAX: return (a < b) ? b : a;
    case ORC_MIN: return (b < a) ? b : a;
    }
    return a;
}

static float ld_f(const void* p, int dtype, size_t i)
{
    if (dtype == ORC_BF16) return orc_bf16_to_f32(((const uint16_t*)p)[i]);
    if (dtype == ORC_F16) return orc_f16_to_f32(((const uint16_t*)p)[i]);
    return ((const float*)p)[i];
}

static void st_f(void* p, int dtype, size_t i, float v)
{
    if (dtype == ORC_BF16)
        ((uint16_t*)p)[i] = orc_f32_to_bf16(v);
    else if (dtype == ORC_F16)
        ((uint16_t*)p)[i] = orc_f32_to_f16(v);
    else
        ((float*)p)[i] = v;
}

/* AVG's final step: one IEEE division of the full fold by N. */
static float finish_f32(int op, float acc, int n)
{
    if (op != ORC_AVG) return acc;
    return MUTANT(2) ? acc * (float)n : acc / (float)n;
}

/* ------------------------------------------------------ ring schedule -- */

/* Chunk that rank r sends at step s of a phase.  Reduce-scatter: step s sends
 * chunk (r - s); all-gather: step s sends chunk (r + 1 - s).  The chunk it
 * receives from its left neighbour is the one that neighbour sends:
 * (r - s - 1) in reduce-scatter and (r - s) in all-gather.
 * [P4] "Ring all-reduce and communication volume", ring_allreduce.py;
 * [P3] section 3, the 4-GPU walkthrough, steps 1 and 2. */
static int send_chunk(int phase, int r, int s, int n)
{
    if (phase == ORC_PHASE_RS) return mod(r - s, n);
    return mod(r + 1 - s + (MUTANT(3) ? 1 : 0), n);
}

/* One step of the ring, for all N ranks at once.  Every rank first puts its
 * outgoing chunk into a message (the isend of a snapshot), then every rank
 * takes its left neighbour's message and, in reduce-scatter, folds it into
 * its own copy of that chunk (received partial on the left), or, in
 * all-gather, overwrites its copy with it.  AVG divides by N in the last
 * reduce-scatter step, where each chunk's fold becomes complete.
 * ev (optional) receives N records, one per sender.
 * [P4] "Ring all-reduce and communication volume" (ring_allreduce.py and the
 * two numbered phase descriptions); [P3] section 3; [P1] s3.2. */
int orc_ring_step(void** bufs, int n, size_t count, int dtype, int op, int phase, int step,
                  orc_event_t* ev)
{
    if (!valid(n, dtype, op) || (phase != ORC_PHASE_RS && phase != ORC_PHASE_AG)) return ORC_EINVAL;
    if (step < 0 || step > n - 2) return ORC_EINVAL;
    size_t C = orc_chunk_size(count, n), es = esize(dtype);
    unsigned char** msg = (unsigned char**)calloc((size_t)n, sizeof *msg);
    if (!msg) return ORC_ENOMEM;
    int rc = ORC_OK;
    for (int r = 0; r < n; ++r) { /* every rank posts its send */
        int k = send_chunk(phase, r, step, n);
        size_t len = orc_chunk_len(count, n, k);
        msg[r] = (unsigned char*)malloc(len * es + 1);
        if (!msg[r]) { rc = ORC_ENOMEM; goto done; }
        memcpy(msg[r], (unsigned char*)bufs[r] + (size_t)k * C * es, len * es);
        if (ev) {
            ev[r].phase = phase;
            ev[r].step = step;
            ev[r].rank = r;
            ev[r].dst = mod(r + 1, n);
            ev[r].send_idx = k;
            ev[r].recv_idx = send_chunk(phase, mod(r - 1, n), step, n);
            ev[r].bytes = (uint64_t)(len * es);
        }
    }
    for (int r = 0; r < n; ++r) { /* every rank receives from its left */
        int left = mod(r - 1, n);
        int k = send_chunk(phase, left, step, n);
        size_t len = orc_chunk_len(count, n, k), off = (size_t)k * C;
        if (phase == ORC_PHASE_AG) {
            memcpy((unsigned char*)bufs[r] + off * es, msg[left], len * es);
            continue;
        }
        int last = (step == n - 2);
        for (size_t j = 0; j < len; ++j) {
            if (dtype == ORC_I32) {
                int32_t got = ((int32_t*)msg[left])[j];
                int32_t* own = (int32_t*)bufs[r] + off + j;
                *own = op_i32(op, got, *own);
            } else {
                float got = ld_f(msg[left], dtype, j);
                float own = ld_f(bufs[r], dtype, off + j);
                float v = MUTANT(4) ? op_f32(op, own, got) : op_f32(op, got, own);
                if (last) v = finish_f32(op, v, n);
                st_f(bufs[r], dtype, off + j, v);
            }
        }
    }
done:
    for (int r = 0; r < n; ++r) free(msg[r]);
    free(msg);
    return rc;
}

/* The full ring all-reduce: N-1 reduce-scatter steps, then N-1 all-gather
 * steps ([P4] "Ring all-reduce and communication volume"; [P3] section 3).
 * trace (optional) receives 2(N-1)*N records in step order; sent (optional)
 * receives the bytes each rank sent, which [P4] counts and [P3] section 4
 * gives in closed form as 2(N-1)/N * S. */
int orc_ring_allreduce(void** bufs, int n, size_t count, int dtype, int op, orc_event_t* trace,
                       uint64_t* sent)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    if (sent) memset(sent, 0, (size_t)n * sizeof *sent);
    orc_event_t* ev = (orc_event_t*)malloc((size_t)n * sizeof *ev);
    if (!ev) return ORC_ENOMEM;
    int nsteps = MUTANT(5) ? n - 2 : n - 1;
    for (int phase = ORC_PHASE_RS; phase <= ORC_PHASE_AG; ++phase) {
        for (int s = 0; s < nsteps; ++s) {
            int rc = orc_ring_step(bufs, n, count, dtype, op, phase, s, ev);
            if (rc != ORC_OK) { free(ev); return rc; }
            for (int r = 0; r < n; ++r) {
                if (sent) sent[r] += ev[r].bytes;
                if (trace) trace[((size_t)phase * (size_t)(n - 1) + (size_t)s) * (size_t)n + (size_t)r] = ev[r];
            }
        }
    }
    free(ev);
    return ORC_OK;
}

/* The same ring, with the N independent transfers of each step run on
 * several host threads (on the ring every link is busy at once, [P3]
 * section 3).  Used only as the timed CPU baseline; the arithmetic and its
 * order are those of orc_ring_step. */
int orc_ring_allreduce_omp(void** bufs, int n, size_t count, int dtype, int op, int nthreads)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    size_t C = orc_chunk_size(count, n), es = esize(dtype);
    unsigned char* msgs = (unsigned char*)malloc((size_t)n * (C ? C : 1) * es);
    if (!msgs) return ORC_ENOMEM;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
    for (int phase = ORC_PHASE_RS; phase <= ORC_PHASE_AG; ++phase) {
        for (int s = 0; s < n - 1; ++s) {
            int last = (phase == ORC_PHASE_RS && s == n - 2);
#pragma omp parallel for schedule(static)
            for (int r = 0; r < n; ++r) {
                int k = send_chunk(phase, r, s, n);
                memcpy(msgs + (size_t)r * C * es, (unsigned char*)bufs[r] + (size_t)k * C * es,
                       orc_chunk_len(count, n, k) * es);
            }
#pragma omp parallel for schedule(static)
            for (int r = 0; r < n; ++r) {
                int left = mod(r - 1, n);
                int k = send_chunk(phase, left, s, n);
                size_t len = orc_chunk_len(count, n, k), off = (size_t)k * C;
                unsigned char* m = msgs + (size_t)(MUTANT(14) ? r : left) * C * es;
                if (phase == ORC_PHASE_AG) {
                    memcpy((unsigned char*)bufs[r] + off * es, m, len * es);
                    continue;
                }
                for (size_t j = 0; j < len; ++j) {
                    if (dtype == ORC_I32) {
                        int32_t* own = (int32_t*)bufs[r] + off + j;
                        *own = op_i32(op, ((int32_t*)m)[j], *own);
                    } else {
                        float v = op_f32(op, ld_f(m, dtype, j), ld_f(bufs[r], dtype, off + j));
                        if (last) v = finish_f32(op, v, n);
                        st_f(bufs[r], dtype, off + j, v);
                    }
                }
            }
        }
    }
    free(msgs);
    return ORC_OK;
}

/* ------------------------------------------------ bf16 wire (compressed) -- */

/* A wire value: what arrives after a transfer in the bf16 wire format. */
static float wire_bf16(float v)
{
    if (MUTANT(11)) return v;
    return orc_bf16_to_f32(orc_f32_to_bf16(v));
}

/* The ring all-reduce of fp32 buffers with a low-precision wire ([P1] s7.3:
 * represent gradients in low precision to cut the communication volume):
 * every chunk that crosses a link is rounded to bf16, while each rank folds in
 * fp32.  Reduce-scatter step s: rank r folds the bf16 image of the partial it
 * receives into its own fp32 copy (received partial on the left); in the last
 * step the owner applies AVG's division and keeps the bf16 image of the
 * result, which is what the all-gather then sends, so every rank ends with
 * the same values.  fp32 buffers, SUM or AVG. */
int orc_ring_allreduce_wire(void** bufs, int n, size_t count, int op)
{
    if (n < 1 || (op != ORC_SUM && op != ORC_AVG)) return ORC_EINVAL;
    size_t C = orc_chunk_size(count, n);
    float* msg = (float*)malloc((size_t)n * (C ? C : 1) * sizeof(float));
    if (!msg) return ORC_ENOMEM;
    for (int phase = ORC_PHASE_RS; phase <= ORC_PHASE_AG; ++phase) {
        for (int s = 0; s < n - 1; ++s) {
            for (int r = 0; r < n; ++r) { /* every rank sends one chunk through the wire */
                int k = send_chunk(phase, r, s, n);
                size_t len = orc_chunk_len(count, n, k);
                for (size_t j = 0; j < len; ++j) {
                    float v = ((float*)bufs[r])[(size_t)k * C + j];
                    msg[(size_t)r * C + j] = phase == ORC_PHASE_RS ? wire_bf16(v) : v;
                }
            }
            for (int r = 0; r < n; ++r) {
                int left = mod(r - 1, n);
                int k = send_chunk(phase, left, s, n);
                size_t len = orc_chunk_len(count, n, k);
                float* own = (float*)bufs[r] + (size_t)k * C;
                for (size_t j = 0; j < len; ++j) {
                    float got = msg[(size_t)left * C + j];
                    if (phase == ORC_PHASE_AG) {
                        own[j] = got; /* already a bf16 image */
                    } else {
                        float v = op_f32(op, got, own[j]);
                        if (s == n - 2) v = wire_bf16(finish_f32(op, v, n));
                        own[j] = v;
                    }
                }
            }
        }
    }
    free(msg);
    return ORC_OK;
}

/* Its result as a definition: element i of chunk c folds
 * acc = x_c; acc = bf16(acc) op x_{c+j} for j = 1..N-1 (the partial is
 * rounded as it is sent, the local value is not), then AVG's division and one
 * last bf16 rounding for the value the all-gather sends.  N = 1 sends
 * nothing and leaves the buffer unchanged. */
int orc_fold_wire(void** bufs, int n, size_t count, int op)
{
    if (n < 1 || (op != ORC_SUM && op != ORC_AVG)) return ORC_EINVAL;
    if (n == 1) return ORC_OK;
    size_t C = orc_chunk_size(count, n);
    for (size_t i = 0; i < count; ++i) {
        int c = (int)(i / C);
        float acc = ((float*)bufs[c])[i];
        for (int j = 1; j < n; ++j) acc = op_f32(op, wire_bf16(acc), ((float*)bufs[mod(c + j, n)])[i]);
        acc = wire_bf16(finish_f32(op, acc, n));
        for (int r = 0; r < n; ++r) ((float*)bufs[r])[i] = acc;
    }
    return ORC_OK;
}

/* ---------------------------------------------------------- double ring -- */

/* The double ring ([P3] section 6: two rings running in opposite directions
 * at once).  Each rank's tensor is cut in two halves, A = [0, H) and
 * B = [H, count) with H = ceil(count / 2); half A is all-reduced by the
 * clockwise ring above (each half chunked on its own: C = ceil(len / N)),
 * half B by the mirror-image ring in which every rank sends to its LEFT
 * neighbour: reduce-scatter step s sends chunk (r + s) to rank r - 1 and
 * receives chunk (r + s + 1) from rank r + 1, so chunk c's partial starts on
 * rank c and gains one rank per hop downwards (c, c-1, c-2, ...), complete
 * on rank c + 1; all-gather step s sends chunk (r - 1 + s) to rank r - 1 and
 * receives chunk (r + s) from rank r + 1.  One step of both rings: */
static int ccw_send_chunk(int phase, int r, int s, int n)
{
    if (phase == ORC_PHASE_RS) return mod(r + s, n);
    return mod(r - 1 + s + (MUTANT(10) ? 1 : 0), n);
}

int orc_double_ring_step(void** bufs, int n, size_t count, int dtype, int op, int phase, int step,
                         uint64_t* sent)
{
    if (!valid(n, dtype, op) || (phase != ORC_PHASE_RS && phase != ORC_PHASE_AG)) return ORC_EINVAL;
    if (step < 0 || step > n - 2) return ORC_EINVAL;
    size_t H = (count + 1) / 2, es = esize(dtype);
    /* half A: the clockwise ring on views of the first H elements */
    int rc = orc_ring_step(bufs, n, H, dtype, op, phase, step, NULL);
    if (rc != ORC_OK) return rc;
    for (int r = 0; r < n && sent; ++r)
        sent[r] += (uint64_t)orc_chunk_len(H, n, send_chunk(phase, r, step, n)) * es;
    /* half B: the counter-clockwise ring */
    size_t cb = count - H, C = orc_chunk_size(cb, n);
    unsigned char** msg = (unsigned char**)calloc((size_t)n, sizeof *msg);
    if (!msg) return ORC_ENOMEM;
    rc = ORC_OK;
    for (int r = 0; r < n; ++r) { /* every rank posts its send to the left */
        int k = ccw_send_chunk(phase, r, step, n);
        size_t len = orc_chunk_len(cb, n, k);
        msg[r] = (unsigned char*)malloc(len * es + 1);
        if (!msg[r]) { rc = ORC_ENOMEM; goto done; }
        memcpy(msg[r], (unsigned char*)bufs[r] + (H + (size_t)k * C) * es, len * es);
        if (sent) sent[r] += (uint64_t)(len * es);
    }
    for (int r = 0; r < n; ++r) { /* every rank receives from its right */
        int right = mod(r + 1, n);
        int k = ccw_send_chunk(phase, right, step, n);
        size_t len = orc_chunk_len(cb, n, k), off = H + (size_t)k * C;
        if (phase == ORC_PHASE_AG) {
            memcpy((unsigned char*)bufs[r] + off * es, msg[right], len * es);
            continue;
        }
        int last = (step == n - 2);
        for (size_t j = 0; j < len; ++j) {
            if (dtype == ORC_I32) {
                int32_t* own = (int32_t*)bufs[r] + off + j;
                *own = op_i32(op, ((int32_t*)msg[right])[j], *own);
            } else {
                float v = op_f32(op, ld_f(msg[right], dtype, j), ld_f(bufs[r], dtype, off + j));
                if (last) v = finish_f32(op, v, n);
                st_f(bufs[r], dtype, off + j, v);
            }
        }
    }
done:
    for (int r = 0; r < n; ++r) free(msg[r]);
    free(msg);
    return rc;
}

/* The whole double ring: N-1 reduce-scatter steps, then N-1 all-gather steps
 * of both rings together; sent (optional) receives the bytes each rank sent
 * (to both neighbours). */
int orc_double_ring_allreduce(void** bufs, int n, size_t count, int dtype, int op, uint64_t* sent)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    if (sent) memset(sent, 0, (size_t)n * sizeof *sent);
    for (int phase = ORC_PHASE_RS; phase <= ORC_PHASE_AG; ++phase)
        for (int s = 0; s < n - 1; ++s) {
            int rc = orc_double_ring_step(bufs, n, count, dtype, op, phase, s, sent);
            if (rc != ORC_OK) return rc;
        }
    return ORC_OK;
}

/* The double ring's result as a plain definition: an element of half A in
 * its half's chunk c folds in ring order c, c+1, ...; an element of half B in
 * chunk c folds downwards c, c-1, c-2, ...; folded in fp32 for every
 * floating dtype and rounded once (its fused one-shot form). */
int orc_fold_double_ring(void** bufs, int n, size_t count, int dtype, int op)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    size_t H = (count + 1) / 2;
    size_t CA = orc_chunk_size(H, n), CB = orc_chunk_size(count - H, n);
    for (size_t i = 0; i < count; ++i) {
        int c, dir;
        if (i < H) { c = (int)(i / CA); dir = 1; }
        else { c = (int)((i - H) / CB); dir = -1; }
        if (dtype == ORC_I32) {
            int32_t acc = ((int32_t*)bufs[c])[i];
            for (int j = 1; j < n; ++j) acc = op_i32(op, acc, ((int32_t*)bufs[mod(c + dir * j, n)])[i]);
            for (int r = 0; r < n; ++r) ((int32_t*)bufs[r])[i] = acc;
        } else {
            float acc = ld_f(bufs[c], dtype, i);
            for (int j = 1; j < n; ++j) acc = op_f32(op, acc, ld_f(bufs[mod(c + dir * j, n)], dtype, i));
            acc = finish_f32(op, acc, n);
            for (int r = 0; r < n; ++r) st_f(bufs[r], dtype, i, acc);
        }
    }
    return ORC_OK;
}

/* ------------------------------------------- one-shot (ring-order fold) -- */

/* The ring's result written as a plain definition.  Following the ring
 * schedule above, chunk c's partial starts on rank c and picks up one rank per
 * hop, so element i of chunk c = i / C is
 *     R[i] = (((x_c[i] op x_{c+1}[i]) op x_{c+2}[i]) ... op x_{c+N-1}[i])
 * with rank indices mod N, then AVG's division.  Every rank receives R.  In a
 * one-shot all-reduce each rank reads every other rank's buffer directly and
 * finishes in one step ([P4] "alpha-beta model", the one-shot/two-shot
 * paragraph).  bf16 values are widened, folded in fp32 and rounded once
 * ([P1] s5.3). */
int orc_fold_ring_order(void** bufs, int n, size_t count, int dtype, int op)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    size_t C = orc_chunk_size(count, n);
    for (size_t i = 0; i < count; ++i) {
        int c = (int)(i / C);
        if (MUTANT(6)) c = mod(c + 1, n);
        if (dtype == ORC_I32) {
            int32_t acc = ((int32_t*)bufs[c])[i];
            for (int j = 1; j < n; ++j) acc = op_i32(op, acc, ((int32_t*)bufs[mod(c + j, n)])[i]);
            for (int r = 0; r < n; ++r) ((int32_t*)bufs[r])[i] = acc;
        } else {
            float acc = ld_f(bufs[c], dtype, i);
            for (int j = 1; j < n; ++j) acc = op_f32(op, acc, ld_f(bufs[mod(c + j, n)], dtype, i));
            acc = finish_f32(op, acc, n);
            for (int r = 0; r < n; ++r) st_f(bufs[r], dtype, i, acc);
        }
    }
    return ORC_OK;
}

/* The same definition on a sample: vals is an [N][m] matrix holding, for m
 * sampled elements, the N ranks' inputs; start[j] is the chunk index of the
 * j-th sampled element (its fold starts on that rank).  out receives m
 * results in the buffers' dtype. */
int orc_fold_samples(const void* vals, int n, size_t m, const int32_t* start, int dtype, int op,
                     void* out)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    for (size_t j = 0; j < m; ++j) {
        int c = start[j];
        if (c < 0 || c >= n) return ORC_EINVAL;
        if (dtype == ORC_I32) {
            const int32_t* v = (const int32_t*)vals;
            int32_t acc = v[(size_t)c * m + j];
            for (int k = 1; k < n; ++k) acc = op_i32(op, acc, v[(size_t)mod(c + k, n) * m + j]);
            ((int32_t*)out)[j] = acc;
        } else {
            float acc = ld_f(vals, dtype, (size_t)c * m + j);
            for (int k = 1; k < n; ++k) acc = op_f32(op, acc, ld_f(vals, dtype, (size_t)mod(c + k, n) * m + j));
            st_f(out, dtype, j, MUTANT(15) ? acc : finish_f32(op, acc, n));
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------ naive all-reduce -- */

/* The naive method: every rank broadcasts its whole tensor to every other
 * rank (an all-gather), then each rank reduces locally, here in rank order
 * 0, 1, ..., N-1 ([P1] s2.1 and s3.1).  Each rank sends (N-1)*S bytes
 * ([P1] s3.3).  Used only as the brute-force cross-check. */
int orc_naive_allreduce(void** bufs, int n, size_t count, int dtype, int op, uint64_t* sent)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    size_t es = esize(dtype);
    unsigned char* gathered = (unsigned char*)malloc((size_t)n * (count ? count : 1) * es);
    if (!gathered) return ORC_ENOMEM;
    for (int r = 0; r < n; ++r) memcpy(gathered + (size_t)r * count * es, bufs[r], count * es);
    for (int r = 0; r < n; ++r) {
        if (sent) sent[r] = (uint64_t)(n - 1) * (uint64_t)(count * es);
        for (size_t i = 0; i < count; ++i) {
            if (dtype == ORC_I32) {
                const int32_t* g = (const int32_t*)gathered;
                int32_t acc = g[i];
                for (int p = 1; p < n; ++p) acc = op_i32(op, acc, g[(size_t)p * count + i]);
                ((int32_t*)bufs[r])[i] = acc;
            } else {
                float acc = ld_f(gathered, dtype, i);
                for (int p = 1; p < n; ++p) acc = op_f32(op, acc, ld_f(gathered, dtype, (size_t)p * count + i));
                st_f(bufs[r], dtype, i, finish_f32(op, acc, n));
            }
        }
    }
    free(gathered);
    return ORC_OK;
}

/* ------------------------------------------------------------------ tree -- */

/* Tree reduction ([P3] section 6): ranks pair up and combine, the pair
 * results pair up again, and after log2 N levels rank 0 holds the reduced
 * value, which is then broadcast back down the tree.  Level l combines
 * x_i <- x_i op x_{i + 2^l} for every i that is a multiple of 2^(l+1) whose
 * partner exists; a rank without a partner (N not a power of two) carries
 * its value up unchanged.  AVG divides at the root in the last level.  Each
 * level's result is stored in the ranks' buffers (bf16 buffers round per
 * level).  The broadcast walks the levels top-down with
 * x_{i + 2^l} <- x_i.  2 * ceil(log2 N) steps. */
int orc_tree_schedule(void** bufs, int n, size_t count, int dtype, int op, int* steps)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    int levels = 0;
    while ((1 << levels) < n) ++levels;
    for (int l = 0; l < levels; ++l) {
        int h = 1 << l, last = (l == levels - 1);
        for (int i = 0; i + h < n; i += 2 * h) {
            for (size_t e = 0; e < count; ++e) {
                if (dtype == ORC_I32) {
                    int32_t* a = (int32_t*)bufs[i] + e;
                    *a = op_i32(op, *a, ((int32_t*)bufs[i + h])[e]);
                } else {
                    float v = op_f32(op, ld_f(bufs[i], dtype, e), ld_f(bufs[i + h], dtype, e));
                    if (last && i == 0) v = finish_f32(op, v, n);
                    st_f(bufs[i], dtype, e, v);
                }
            }
        }
    }
    for (int l = levels - 1; l >= 0; --l) {
        int h = 1 << l;
        for (int i = 0; i + h < n; i += 2 * h)
            memcpy(bufs[i + h], bufs[i], count * esize(dtype));
    }
    if (steps) *steps = 2 * levels;
    return ORC_OK;
}

/* The tree's result as a plain definition, folded in fp32 for every dtype
 * with floating values and rounded once (the fused tree-order one-shot):
 * per element, the same pairwise levels as orc_tree_schedule on a private
 * copy of the N values, then AVG's division, then store to every rank. */
int orc_tree_fold(void** bufs, int n, size_t count, int dtype, int op)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    float* v = (float*)malloc((size_t)n * sizeof *v);
    int32_t* w = (int32_t*)malloc((size_t)n * sizeof *w);
    char* alive = (char*)malloc((size_t)n);
    if (!v || !w || !alive) { free(v); free(w); free(alive); return ORC_ENOMEM; }
    for (size_t e = 0; e < count; ++e) {
        for (int r = 0; r < n; ++r) {
            if (dtype == ORC_I32) w[r] = ((int32_t*)bufs[r])[e];
            else v[r] = ld_f(bufs[r], dtype, e);
            alive[r] = 1;
        }
        for (int h = 1; h < n; h *= 2) {
            for (int i = 0; i + h < n; i += 2 * h) {
                if (!alive[i + h]) continue;
                if (dtype == ORC_I32) w[i] = op_i32(op, w[i], w[i + h]);
                else v[i] = op_f32(op, v[i], v[i + h]);
            }
            if (MUTANT(13)) {  /* the unpaired rank joins the pair before it at this level */
                int i = ((n - 1) / (2 * h)) * (2 * h);
                if (i + h >= n && i > 0 && alive[i]) {
                    if (dtype == ORC_I32) w[i - 2 * h] = op_i32(op, w[i - 2 * h], w[i]);
                    else v[i - 2 * h] = op_f32(op, v[i - 2 * h], v[i]);
                    alive[i] = 0;
                }
            }
        }
        for (int r = 0; r < n; ++r) {
            if (dtype == ORC_I32) ((int32_t*)bufs[r])[e] = w[0];
            else st_f(bufs[r], dtype, e, finish_f32(op, v[0], n));
        }
    }
    free(v);
    free(w);
    free(alive);
    return ORC_OK;
}

/* --------------------------------------- reduce-scatter, gather, a2a -- */

/* Reduce-scatter ([P4] "The five primitives": reduce, then split into N
 * parts, rank r gets part r; [P3] section 6: the ring's first phase used on
 * its own).  Part r is chunk r of the inputs; its value is the same
 * ring-order fold as the all-reduce's (starting on rank r), so a
 * reduce-scatter followed by an all-gather equals the all-reduce bit for
 * bit.  send[p] holds N*recvcount elements, recv[r] holds recvcount. */
int orc_reduce_scatter(const void* const* send, void* const* recv, int n, size_t recvcount, int dtype,
                       int op)
{
    if (!valid(n, dtype, op)) return ORC_EINVAL;
    for (int r = 0; r < n; ++r) {
        int start = MUTANT(7) ? mod(r + 1, n) : r;
        for (size_t i = 0; i < recvcount; ++i) {
            size_t e = (size_t)r * recvcount + i;
            if (dtype == ORC_I32) {
                int32_t acc = ((const int32_t*)send[start])[e];
                for (int j = 1; j < n; ++j) acc = op_i32(op, acc, ((const int32_t*)send[mod(start + j, n)])[e]);
                ((int32_t*)recv[r])[i] = acc;
            } else {
                float acc = ld_f(send[start], dtype, e);
                for (int j = 1; j < n; ++j) acc = op_f32(op, acc, ld_f(send[mod(start + j, n)], dtype, e));
                st_f(recv[r], dtype, i, finish_f32(op, acc, n));
            }
        }
    }
    return ORC_OK;
}

/* All-gather ([P4] "The five primitives"): every rank contributes one part
 * and every rank receives all parts concatenated in rank order:
 * recv[r][p*C + i] = send[p][i]. */
int orc_all_gather(const void* const* send, void* const* recv, int n, size_t sendcount, int dtype)
{
    if (!valid(n, dtype, ORC_SUM)) return ORC_EINVAL;
    size_t es = esize(dtype);
    for (int r = 0; r < n; ++r)
        for (int p = 0; p < n; ++p) {
            int src = MUTANT(8) ? mod(p + 1, n) : p;
            memcpy((unsigned char*)recv[r] + (size_t)p * sendcount * es, send[src], sendcount * es);
        }
    return ORC_OK;
}

/* All-to-all ([P4] "The five primitives": rank r's p-th block goes to rank
 * p, a transpose): recv[r][p*C + i] = send[p][r*C + i]. */
int orc_all_to_all(const void* const* send, void* const* recv, int n, size_t count_per_peer, int dtype)
{
    if (!valid(n, dtype, ORC_SUM)) return ORC_EINVAL;
    size_t es = esize(dtype), b = count_per_peer * es;
    for (int r = 0; r < n; ++r)
        for (int p = 0; p < n; ++p) {
            size_t blk = MUTANT(9) ? (size_t)p : (size_t)r;
            memcpy((unsigned char*)recv[r] + (size_t)p * b, (const unsigned char*)send[p] + blk * b, b);
        }
    return ORC_OK;
}

/* -------------------------------------------------------------- buckets -- */

/* DDP-style bucket plan ([P2] s3.3: gradients are put into buckets in the
 * order given and a bucket is handed to the all-reduce once its gradients
 * reach the threshold; [P1] s5.2: bucket_cap_mb, default 25).  Greedy, never
 * splits a tensor: each tensor joins the open bucket, and the bucket closes
 * as soon as its bytes reach cap_bytes.  A tensor at least as large as the
 * cap therefore ends the bucket it joins.  Outputs, per tensor, its bucket
 * and its element offset inside the bucket. */
int orc_bucket_plan(const uint64_t* numels, int nt, uint64_t elem_bytes, uint64_t cap_bytes,
                    int32_t* bucket_of, uint64_t* offset_of, int32_t* nbuckets)
{
    if (nt < 0 || elem_bytes == 0) return ORC_EINVAL;
    int32_t b = 0;
    uint64_t off = 0, bytes = 0;
    int open = 0;
    for (int t = 0; t < nt; ++t) {
        bucket_of[t] = b;
        offset_of[t] = off;
        off += numels[t];
        bytes += numels[t] * elem_bytes;
        open = 1;
        if (bytes >= cap_bytes) {
            ++b;
            off = 0;
            bytes = 0;
            open = 0;
        }
    }
    *nbuckets = b + open;
    return ORC_OK;
}

/* Bucket pack for one rank: bucket[offset_of[t] + j] = widen(grad[t][j]) for
 * every tensor t of the bucket (bf16 -> fp32 is exact; [P1] s5.3 reduce
 * low-precision gradients in fp32).  grads[t] is NULL for tensors outside
 * the bucket. */
int orc_bucket_pack(const void* const* grads, const uint64_t* numels, const int32_t* bucket_of,
                    const uint64_t* offset_of, int nt, int bucket, int grad_dtype, float* out)
{
    for (int t = 0; t < nt; ++t) {
        if (bucket_of[t] != bucket) continue;
        for (uint64_t j = 0; j < numels[t]; ++j) out[offset_of[t] + j] = ld_f(grads[t], grad_dtype, j);
    }
    return ORC_OK;
}

/* Bucket unpack for one rank: grad[t][j] = round(bucket[offset + j] / N) for
 * AVG, round(bucket[offset + j]) for SUM, with one round-to-nearest-even to
 * the gradient dtype. */
int orc_bucket_unpack(void* const* grads, const uint64_t* numels, const int32_t* bucket_of,
                      const uint64_t* offset_of, int nt, int bucket, int grad_dtype, const float* in,
                      int n, int op)
{
    if (op != ORC_SUM && op != ORC_AVG) return ORC_EINVAL;
    for (int t = 0; t < nt; ++t) {
        if (bucket_of[t] != bucket) continue;
        for (uint64_t j = 0; j < numels[t]; ++j)
            st_f(grads[t], grad_dtype, j, finish_f32(op, in[offset_of[t] + j], n));
    }
    return ORC_OK;
}
