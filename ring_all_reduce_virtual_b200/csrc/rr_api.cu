// rr_api.cu -- the C ABI (include/rr.h): argument checks, the ring and tree
// schedules as launch tables, the per-size picker, bucket plans, call
// statistics.  Host code only; every data movement runs in the kernels.
//
// Sources, cited by tag in the comments below:
//   [P1] "How all-reduce keeps every card identical" (mhpq.cn, news 451051)
//   [P2] "AllReduce from principle to tuning" (xxqk.cn, news 376101)
//   [P3] "Training gradient sync and collective communication: from parameter
//        server to Ring AllReduce" (geek-doc.cn)
//   [P4] "Collective communication primitives" (ai-infra-handbooks)
#include <algorithm>
#include <atomic>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "rr.h"
#include "rr_internal.h"
#include "rr_picker_table.h"

using namespace rr;

struct rr_bucket_plan {
    int ntensors = 0;
    int grad_dtype = RR_BF16;
    size_t cap_bytes = 0;
    std::vector<uint64_t> numel;   // per tensor
    std::vector<uint64_t> offset;  // per tensor: element offset in its bucket
    std::vector<int> bucket_of;    // per tensor
    std::vector<int> first;        // per bucket: first tensor
    std::vector<int> count;        // per bucket: number of tensors
    std::vector<uint64_t> bnumel;  // per bucket: elements
};

namespace {

thread_local rr_stats_t t_stats{};
thread_local std::string t_error;

// Picker parameters: the sweep's alpha-beta fit until rr_set_picker_params
// (from any thread) sets others, which also switches AUTO from the measured
// table to the model.
std::atomic<double> g_launch_s{kPickerAlphaS};   // cost of one launch
std::atomic<double> g_hbm_bps{kPickerBetaBps};   // effective HBM bytes/s
std::atomic<bool> g_use_model{false};

rr_status_t fail(rr_status_t st, const std::string& why)
{
    t_error = why;
    return st;
}

rr_status_t cuda_fail(cudaError_t e, const char* where)
{
    t_error = std::string(where) + ": " + cudaGetErrorString(e);
    return RR_ERR_CUDA;
}

bool env_flag(const char* name)
{
    const char* v = std::getenv(name);
    return v && *v && std::strcmp(v, "0") != 0;
}

size_t esize(rr_dtype_t d) { return d == RR_BF16 || d == RR_F16 ? 2u : 4u; }

bool dtype_ok(rr_dtype_t d) { return d == RR_F32 || d == RR_BF16 || d == RR_I32 || d == RR_F16; }
bool op_ok(rr_op_t o) { return o >= RR_SUM && o <= RR_PROD; }

const char* algo_name(int a)
{
    switch (a) {
    case RR_ALGO_AUTO: return "auto";
    case RR_ALGO_RING: return "ring";
    case RR_ALGO_ONESHOT: return "oneshot";
    case RR_ALGO_TREE: return "tree";
    case RR_ALGO_TREE_ONESHOT: return "tree_oneshot";
    case RR_ALGO_TWO_SHOT: return "two_shot";
    case RR_ALGO_DOUBLE_RING: return "double_ring";
    }
    return "?";
}

// Common checks of dtype, op and rank count.
rr_status_t check_basic(int n, rr_dtype_t dtype, rr_op_t op)
{
    if (n < 1 || n > RR_MAX_RANKS) return fail(RR_ERR_INVALID_ARG, "nranks must be in 1..64");
    if (!dtype_ok(dtype)) return fail(RR_ERR_INVALID_ARG, "unknown dtype");
    if (!op_ok(op)) return fail(RR_ERR_INVALID_ARG, "unknown op");
    if (dtype == RR_I32 && op == RR_AVG) return fail(RR_ERR_UNSUPPORTED, "AVG is not defined for int32");
    return RR_OK;
}

// Element counts above 2^48 (far beyond any device memory) are refused, so
// count * 64 ranks * 4 bytes stays below 2^56 and no byte range wraps.
constexpr uint64_t kMaxElems = 1ull << 48;

rr_status_t check_count(uint64_t count)
{
    if (count > kMaxElems) return fail(RR_ERR_INVALID_ARG, "element count above 2^48");
    return RR_OK;
}

struct Span {
    uintptr_t lo, hi;
    bool out;
};

// The spans of a call with one or two buffers per rank, kept on the stack so
// that a call allocates nothing on the host either.
struct SpanBuf {
    Span s[2 * RR_MAX_RANKS];
    size_t n = 0;
    void push_back(const Span& x) { s[n++] = x; }
    Span* begin() { return s; }
    Span* end() { return s + n; }
    size_t size() const { return n; }
    Span& operator[](size_t i) { return s[i]; }
};

// Every output span must be non-NULL and overlap no other span; inputs may
// overlap one another (they are only read).
template <class Spans>
rr_status_t check_spans(Spans& s)
{
    for (const Span& a : s)
        if (a.lo == 0) return fail(RR_ERR_INVALID_ARG, "NULL buffer pointer");
    std::sort(s.begin(), s.end(), [](const Span& a, const Span& b) { return a.lo < b.lo; });
    for (size_t i = 0; i < s.size(); ++i)
        for (size_t j = i + 1; j < s.size() && s[j].lo < s[i].hi; ++j)
            if (s[i].out || s[j].out) return fail(RR_ERR_INVALID_ARG, "buffers overlap (or repeat)");
    return RR_OK;
}

// Every pointer on a boundary of its element size (a device access of an
// element at any other address faults).
rr_status_t check_elem_aligned(const void* const* p, int n, size_t es)
{
    for (int i = 0; i < n; ++i)
        if ((uintptr_t)p[i] % es != 0) return fail(RR_ERR_INVALID_ARG, "buffer not aligned to its element size");
    return RR_OK;
}

// True when all pointers agree modulo 16 bytes.
bool same_phase(const void* const* p, int n)
{
    for (int i = 1; i < n; ++i)
        if (((uintptr_t)p[i] & 15u) != ((uintptr_t)p[0] & 15u)) return false;
    return true;
}

// Optional (RR_DEBUG=1): reject pointers the driver does not know as device
// or managed memory, before any launch.
rr_status_t check_device_ptrs(const void* const* p, int n)
{
    static const bool debug = env_flag("RR_DEBUG");  // read once: getenv scans the environment
    if (!debug) return RR_OK;
    for (int i = 0; i < n; ++i) {
        cudaPointerAttributes a{};
        if (cudaPointerGetAttributes(&a, p[i]) != cudaSuccess ||
            (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged)) {
            cudaGetLastError();
            return fail(RR_ERR_INVALID_ARG, "pointer is not device memory");
        }
    }
    return RR_OK;
}

// Optional (RR_DEBUG=1): after a call that enqueued work, synchronise its
// stream (unless the stream is being captured into a graph) and report a
// kernel fault, or a bounded device wait that ran out, at the call that
// caused it instead of at some later synchronisation.
rr_status_t debug_check(rr_status_t st, cudaStream_t stream)
{
    static const bool debug = env_flag("RR_DEBUG");
    if (!debug || st != RR_OK || t_stats.launches == 0) return st;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
        cudaGetLastError();
        return st;
    }
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e, "RR_DEBUG: the call's kernels failed");
    unsigned int ran_out = 0, in_flight = 0;
    if ((e = take_bulk_timeouts(&ran_out, &in_flight)) != cudaSuccess) return cuda_fail(e, "RR_DEBUG: reading the wait counters");
    if (ran_out || in_flight)
        return fail(RR_ERR_TIMEOUT, "RR_DEBUG: bounded device waits ran out on " + std::to_string(ran_out) +
                                        " tiles during this call; copies not seen to land: " + std::to_string(in_flight));
    return st;
}

uint64_t ceil_div(uint64_t a, uint64_t b) { return b ? (a + b - 1) / b : 0; }

uint64_t chunk_len(uint64_t count, int n, int k)
{
    const uint64_t C = ceil_div(count, (uint64_t)n), lo = (uint64_t)k * C;
    if (lo >= count) return 0;
    return std::min(C, count - lo);
}

int imod(int a, int n) { return ((a % n) + n) % n; }

// Ring schedule ([P4] "Ring all-reduce and communication volume",
// ring_allreduce.py; [P3] section 3, steps 1-2 of the 4-GPU walkthrough):
// at reduce-scatter step s rank r sends chunk (r - s) and receives chunk
// (r - s - 1) from its left neighbour; at all-gather step s it sends
// (r + 1 - s) and receives (r - s).
int ring_send_chunk(int phase, int r, int s, int n)
{
    return phase == RR_PHASE_REDUCE_SCATTER ? imod(r - s, n) : imod(r + 1 - s, n);
}

// The mirror-image ring of the double ring ([P3] section 6): every rank sends
// to its left neighbour.  Reduce-scatter step s sends chunk (r + s) and
// receives chunk (r + s + 1) from the right; all-gather step s sends chunk
// (r - 1 + s) and receives (r + s).  Chunk c's partial starts on rank c and
// gains one rank per hop downwards; it is complete on rank c + 1.
int ccw_send_chunk(int phase, int r, int s, int n)
{
    return phase == RR_PHASE_REDUCE_SCATTER ? imod(r + s, n) : imod(r - 1 + s, n);
}

void log_call(const char* what, int n, size_t count, rr_dtype_t dtype, int op, int algo)
{
    static const bool on = env_flag("RR_LOG");
    if (on)
        std::fprintf(stderr, "[rr] %s nranks=%d count=%zu dtype=%d op=%d algo=%s launches=%d\n", what, n,
                     count, (int)dtype, op, algo_name(algo), t_stats.launches);
}

void stats_begin(int algo, int n, uint64_t S)
{
    t_stats = rr_stats_t{};
    t_stats.algo = algo;
    t_stats.nranks = n;
    t_stats.bytes_per_rank = S;
}

uint64_t now_ns()
{
    return (uint64_t)std::chrono::duration_cast<std::chrono::nanoseconds>(
               std::chrono::steady_clock::now().time_since_epoch())
        .count();
}

// One API call: an NVTX range named for it (for timeline tools; a no-op
// when none is attached), and its host time, entry to return, into the
// call's statistics.
struct CallTimer {
    uint64_t t0;
    explicit CallTimer(const char* name)
    {
        nvtxRangePushA(name);
        t0 = now_ns();
    }
    ~CallTimer()
    {
        t_stats.host_ns = now_ns() - t0;
        nvtxRangePop();
    }
};

// An NVTX range around one launch of a step-by-step schedule.
struct StepRange {
    StepRange(const char* what, int phase, int step)
    {
        char name[64];
        std::snprintf(name, sizeof name, "%s %s step %d", what, phase == RR_PHASE_REDUCE_SCATTER ? "RS" : "AG", step);
        nvtxRangePushA(name);
    }
    ~StepRange() { nvtxRangePop(); }
};

// A launch, its host time added to the call's statistics.
template <class F>
cudaError_t timed_launch(F&& f)
{
    const uint64_t t0 = now_ns();
    const cudaError_t e = f();
    t_stats.launch_ns += now_ns() - t0;
    return e;
}

// Build and launch one ring step (all ranks at once).
rr_status_t ring_step_launch(void* const* bufs, int n, size_t count, rr_dtype_t dtype, rr_op_t op, int phase,
                             int step, cudaStream_t stream, bool wire = false)
{
    const size_t es = esize(dtype);
    const uint64_t C = ceil_div(count, (uint64_t)n);
    StepParams p{};
    p.nseg = n;
    p.nin = phase == RR_PHASE_REDUCE_SCATTER ? 2 : 1;
    p.vec_ok = same_phase(bufs, n);
    p.divisor = (float)n;
    uint64_t maxlen = 0;
    for (int r = 0; r < n; ++r) {
        const int left = imod(r - 1, n);
        const int k = ring_send_chunk(phase, left, step, n);  // the chunk r receives
        const uint64_t lo = (uint64_t)k * C, len = chunk_len(count, n, k);
        p.seg[r].in0 = static_cast<const char*>(bufs[left]) + lo * es;
        p.seg[r].in1 = p.nin == 2 ? static_cast<const char*>(bufs[r]) + lo * es : nullptr;
        p.seg[r].out = static_cast<char*>(bufs[r]) + lo * es;
        p.seg[r].len = len;
        maxlen = std::max(maxlen, len);
    }
    p.tps = std::max<uint64_t>(1, ceil_div(maxlen, tile_elems(dtype, kVptMove)));
    // AVG divides once, in the step that completes each chunk's fold
    int op_eff = op;
    if (op == RR_AVG && !(phase == RR_PHASE_REDUCE_SCATTER && step == n - 2)) op_eff = RR_SUM;
    if (maxlen == 0) return RR_OK;
    const StepRange range("ring", phase, step);
    cudaError_t e;
    if (wire && p.nin == 2)  // a bf16-wire reduce-scatter step; the all-gather copies wire values
        e = timed_launch([&] { return launch_step_wire(op_eff, step == n - 2 ? 1 : 2, p, stream); });
    else
        e = timed_launch([&] { return launch_step(dtype, op_eff, p, stream); });
    if (e != cudaSuccess) return cuda_fail(e, "ring step launch");
    t_stats.launches += 1;
    return RR_OK;
}

// The ring schedule in one launch (ring_chain_kernel: every tile of every
// chunk carried through the 2(N-1) steps by one CTA) when every buffer is at
// the same 16-byte phase; otherwise one launch per step.  wire: the bf16 wire
// format (fp32 buffers).
rr_status_t run_ring(void* const* bufs, int n, size_t count, rr_dtype_t dtype, rr_op_t op, cudaStream_t stream,
                     bool wire = false)
{
    const size_t es = esize(dtype);
    if (same_phase(bufs, n)) {
        ChainParams p{};
        for (int r = 0; r < n; ++r) p.buf[r] = bufs[r];
        p.n = n;
        p.vec_ok = 1;
        p.divisor = (float)n;
        p.nhalf = 1;
        p.count = count;
        p.H = count;
        p.C[0] = ceil_div(count, (uint64_t)n);
        p.tps = std::max<uint64_t>(1, ceil_div(p.C[0], chain_tile_elems(dtype)));
        cudaError_t e = timed_launch([&] { return launch_ring_chain(dtype, op, wire, p, stream); });
        if (e != cudaSuccess) return cuda_fail(e, "ring launch");
        t_stats.launches += 1;
    } else {
        for (int phase = RR_PHASE_REDUCE_SCATTER; phase <= RR_PHASE_ALL_GATHER; ++phase)
            for (int s = 0; s < n - 1; ++s) {
                rr_status_t st = ring_step_launch(bufs, n, count, dtype, op, phase, s, stream, wire);
                if (st != RR_OK) return st;
            }
    }
    // over the reduce-scatter rank r sends chunks r, r-1, ..., r+2 (every chunk
    // but r+1), over the all-gather chunks r+1, r, ..., r+3 (every chunk but r+2)
    const uint64_t wes = wire ? 2 : es;  // bytes a sent element takes on the wire
    for (int r = 0; r < n; ++r) {
        const uint64_t sent =
            (2 * (uint64_t)count - chunk_len(count, n, imod(r + 1, n)) - chunk_len(count, n, imod(r + 2, n))) * wes;
        t_stats.bytes_sent_max = std::max<uint64_t>(t_stats.bytes_sent_max, sent);
        t_stats.bytes_sent_total += sent;
    }
    t_stats.steps = 2 * (n - 1);
    // each reduce-scatter step reads 2 and writes 1 chunk per rank, each
    // all-gather step reads and writes 1: 5 (N-1) S in all
    t_stats.hbm_bytes = 5ull * (uint64_t)(n - 1) * count * es;
    return RR_OK;
}

// One step of both rings of the double ring, one launch: segments 0..N-1 are
// the clockwise ring on the first half [0, H), segments N..2N-1 the
// counter-clockwise ring on the second half [H, count).
rr_status_t double_ring_step_launch(void* const* bufs, int n, size_t count, rr_dtype_t dtype, rr_op_t op,
                                    int phase, int step, cudaStream_t stream, std::vector<uint64_t>& sent)
{
    const size_t es = esize(dtype);
    const uint64_t H = (count + 1) / 2, cb = count - H;
    const uint64_t CA = ceil_div(H, (uint64_t)n), CB = ceil_div(cb, (uint64_t)n);
    StepParams p{};
    p.nseg = 2 * n;
    p.nin = phase == RR_PHASE_REDUCE_SCATTER ? 2 : 1;
    p.vec_ok = same_phase(bufs, n);
    p.divisor = (float)n;
    uint64_t maxlen = 0;
    for (int r = 0; r < n; ++r) {
        const int left = imod(r - 1, n), right = imod(r + 1, n);
        const int ka = ring_send_chunk(phase, left, step, n);  // half A, from the left
        const uint64_t la = (uint64_t)ka * CA, na = chunk_len(H, n, ka);
        p.seg[r] = {static_cast<const char*>(bufs[left]) + la * es,
                    p.nin == 2 ? static_cast<const char*>(bufs[r]) + la * es : nullptr,
                    static_cast<char*>(bufs[r]) + la * es, na};
        const int kb = ccw_send_chunk(phase, right, step, n);  // half B, from the right
        const uint64_t lb = H + (uint64_t)kb * CB, nb = chunk_len(cb, n, kb);
        p.seg[n + r] = {static_cast<const char*>(bufs[right]) + lb * es,
                        p.nin == 2 ? static_cast<const char*>(bufs[r]) + lb * es : nullptr,
                        static_cast<char*>(bufs[r]) + lb * es, nb};
        maxlen = std::max(maxlen, std::max(na, nb));
        sent[r] += (chunk_len(H, n, ring_send_chunk(phase, r, step, n)) +
                    chunk_len(cb, n, ccw_send_chunk(phase, r, step, n))) * es;
    }
    p.tps = std::max<uint64_t>(1, ceil_div(maxlen, tile_elems(dtype, kVptMove)));
    int op_eff = op;
    if (op == RR_AVG && !(phase == RR_PHASE_REDUCE_SCATTER && step == n - 2)) op_eff = RR_SUM;
    if (maxlen == 0) return RR_OK;
    const StepRange range("double ring", phase, step);
    cudaError_t e = timed_launch([&] { return launch_step(dtype, op_eff, p, stream); });
    if (e != cudaSuccess) return cuda_fail(e, "double ring step launch");
    t_stats.launches += 1;
    return RR_OK;
}

rr_status_t run_double_ring(void* const* bufs, int n, size_t count, rr_dtype_t dtype, rr_op_t op,
                            cudaStream_t stream)
{
    std::vector<uint64_t> sent(n, 0);
    if (same_phase(bufs, n)) {  // both rings in one launch (ring_chain_kernel, two halves)
        const uint64_t H = (count + 1) / 2, cb = count - H;
        ChainParams p{};
        for (int r = 0; r < n; ++r) p.buf[r] = bufs[r];
        p.n = n;
        p.vec_ok = 1;
        p.divisor = (float)n;
        p.nhalf = 2;
        p.count = count;
        p.H = H;
        p.C[0] = ceil_div(H, (uint64_t)n);
        p.C[1] = ceil_div(cb, (uint64_t)n);
        p.tps = std::max<uint64_t>(1, ceil_div(std::max(p.C[0], p.C[1]), chain_tile_elems(dtype)));
        cudaError_t e = timed_launch([&] { return launch_ring_chain(dtype, op, false, p, stream); });
        if (e != cudaSuccess) return cuda_fail(e, "double ring launch");
        t_stats.launches += 1;
        // each half as the ring: the clockwise half skips chunks r+1 and r+2, the
        // mirror ring (chunks sent downwards) chunks r-1 and r-2
        for (int r = 0; r < n; ++r)
            sent[r] = (2 * H - chunk_len(H, n, imod(r + 1, n)) - chunk_len(H, n, imod(r + 2, n)) + 2 * cb -
                       chunk_len(cb, n, imod(r - 1, n)) - chunk_len(cb, n, imod(r - 2, n))) * esize(dtype);
    } else {
        for (int phase = RR_PHASE_REDUCE_SCATTER; phase <= RR_PHASE_ALL_GATHER; ++phase)
            for (int s = 0; s < n - 1; ++s) {
                rr_status_t st = double_ring_step_launch(bufs, n, count, dtype, op, phase, s, stream, sent);
                if (st != RR_OK) return st;
            }
    }
    t_stats.steps = 2 * (n - 1);
    for (int r = 0; r < n; ++r) {
        t_stats.bytes_sent_max = std::max<uint64_t>(t_stats.bytes_sent_max, sent[r]);
        t_stats.bytes_sent_total += sent[r];
    }
    t_stats.hbm_bytes = 5ull * (uint64_t)(n - 1) * count * esize(dtype);
    return RR_OK;
}

int tree_levels(int n)
{
    int l = 0;
    while ((1 << l) < n) ++l;
    return l;
}

// Tree schedule ([P3] section 6): pairwise reduce levels up to rank 0, then
// broadcast levels back down.
rr_status_t run_tree(void* const* bufs, int n, size_t count, rr_dtype_t dtype, rr_op_t op, cudaStream_t stream)
{
    const size_t es = esize(dtype);
    const int L = tree_levels(n);
    const bool vec = same_phase(bufs, n);
    std::vector<uint64_t> sent(n, 0);
    uint64_t pairs_total = 0;
    if (vec) {  // every level in one launch (tree_chain_kernel)
        ChainParams p{};
        for (int r = 0; r < n; ++r) p.buf[r] = bufs[r];
        p.n = n;
        p.vec_ok = 1;
        p.divisor = (float)n;
        p.count = count;
        p.H = count;
        p.tps = std::max<uint64_t>(1, ceil_div(count, chain_tile_elems(dtype)));
        cudaError_t e = timed_launch([&] { return launch_tree_chain(dtype, op, p, stream); });
        if (e != cudaSuccess) return cuda_fail(e, "tree launch");
        t_stats.launches += 1;
    }
    for (int pass = 0; pass < 2; ++pass) {
        for (int i = 0; i < L; ++i) {
            const int l = pass == 0 ? i : L - 1 - i;
            const int h = 1 << l;
            StepParams p{};
            p.nin = pass == 0 ? 2 : 1;
            p.vec_ok = vec;
            p.divisor = (float)n;
            p.tps = std::max<uint64_t>(1, ceil_div(count, tile_elems(dtype, kVptMove)));
            for (int a = 0; a + h < n; a += 2 * h) {
                StepSeg& sg = p.seg[p.nseg++];
                if (pass == 0) {  // x_a <- x_a op x_{a+h}
                    sg.in0 = bufs[a];
                    sg.in1 = bufs[a + h];
                    sg.out = bufs[a];
                    sent[a + h] += count * es;
                } else {          // x_{a+h} <- x_a
                    sg.in0 = bufs[a];
                    sg.out = bufs[a + h];
                    sent[a] += count * es;
                }
                sg.len = count;
                ++pairs_total;
            }
            if (vec) continue;  // counted only: the levels ran in the one launch above
            int op_eff = op;
            if (op == RR_AVG && !(pass == 0 && l == L - 1)) op_eff = RR_SUM;
            cudaError_t e = timed_launch([&] { return launch_step(dtype, op_eff, p, stream); });
            if (e != cudaSuccess) return cuda_fail(e, "tree level launch");
            t_stats.launches += 1;
        }
    }
    t_stats.steps = 2 * L;
    for (int r = 0; r < n; ++r) {
        t_stats.bytes_sent_max = std::max<uint64_t>(t_stats.bytes_sent_max, sent[r]);
        t_stats.bytes_sent_total += sent[r];
    }
    // reduce: 3 S per pair, broadcast: 2 S per pair, N-1 pairs each way
    t_stats.hbm_bytes = 5ull * (pairs_total / 2) * count * es;
    return RR_OK;
}

rr_status_t run_rank_kernel(int kind, const void* const* in, void* const* out, int n, uint64_t C,
                            uint64_t count, uint64_t nseg, uint64_t tps, rr_dtype_t dtype, int op, bool vec,
                            cudaStream_t stream, uint64_t lo = 0, uint64_t hi = UINT64_MAX, bool owner_only = false)
{
    RankParams p{};
    for (int r = 0; r < n; ++r) {
        p.in[r] = in[r];
        p.out[r] = out[r];
    }
    p.n = n;
    p.vec_ok = vec;
    p.divisor = (float)n;
    p.C = C;
    p.count = count;
    p.nseg = nseg;
    p.tps = tps;
    p.lo = lo;
    p.hi = hi;
    p.owner_only = owner_only ? 1 : 0;
    p.waits = bulk_wait_counters();  // looked up once per launch
    cudaError_t e = timed_launch([&] { return launch_rank_kernel(kind, dtype, op, p, stream); });
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    t_stats.launches += 1;
    return RR_OK;
}

// Alignment class of a call's buffers, as the picker's table keys it: 0 all
// 16-byte aligned, 1 all at one other 16-byte phase, 2 phases that differ.
int align_class(const void* const* p, int n)
{
    if (!same_phase(p, n)) return 2;
    return ((uintptr_t)p[0] & 15u) ? 1 : 0;
}

int log2_round(double x) { return x <= 1 ? 0 : (int)std::lround(std::log2(x)); }

// The alpha-beta model of [P3] section 4 on one GPU: every "link" is HBM, a
// step costs one launch, and its bytes are the HBM bytes it reads and writes
// (ring 5(N-1) S over 2(N-1) launches -- one launch when the buffers share a
// phase, but the model keeps the schedule's steps --, one-shot 2 N S in one,
// two-shot (2N+1) S in two).  bf16 and fp16 always take ONESHOT: the ring
// rounds its 16-bit partials at every hop, the fp32-accumulating one-shot
// does not ([P1] s5.3).
rr_algo_t model_pick(int nranks, size_t count, rr_dtype_t dtype)
{
    if (dtype == RR_BF16 || dtype == RR_F16 || nranks <= 1) return RR_ALGO_ONESHOT;
    const double n = nranks, S = (double)count * (double)esize(dtype);
    const double alpha = g_launch_s.load(), beta = g_hbm_bps.load();
    const double ring = 2 * (n - 1) * alpha + 5 * (n - 1) * S / beta;
    const double one = alpha + 2 * n * S / beta;
    const double two = 2 * alpha + (2 * n + 1) * S / beta;
    if (ring < one && ring < two) return RR_ALGO_RING;
    return two < one ? RR_ALGO_TWO_SHOT : RR_ALGO_ONESHOT;
}

// The measured table's choice for (N, bytes per rank, alignment class): among
// the points measured in that class (the aligned class if the table has none
// of it), the nearest measured rank count (in log2 ratio; the smaller on a
// tie), then the nearest measured size there.  RR_ALGO_AUTO if the table is
// empty.
rr_algo_t table_pick(int n, uint64_t bytes, int align)
{
    bool have = false;
    for (const PickerPoint& e : kPickerTable) have = have || e.align == align;
    if (!have) align = 0;
    const int lb = log2_round((double)bytes);
    double best_dn = 1e30;
    int best_n = 0;
    for (const PickerPoint& e : kPickerTable) {
        if (e.align != align) continue;
        const double dn = std::fabs(std::log2((double)e.nranks / (double)n));
        if (dn < best_dn - 1e-12 || (std::fabs(dn - best_dn) <= 1e-12 && e.nranks < best_n)) {
            best_dn = dn;
            best_n = e.nranks;
        }
    }
    int best_d = 1 << 30;
    rr_algo_t pick = RR_ALGO_AUTO;
    for (const PickerPoint& e : kPickerTable) {
        if (e.nranks != best_n || e.align != align) continue;
        const int d = std::abs(e.log2_bytes - lb);
        if (d < best_d) {
            best_d = d;
            pick = (rr_algo_t)e.algo;
        }
    }
    return pick;
}

// AUTO's choice for a call on these buffers.  bf16 and fp16 never take RING
// (its partials would be rounded at every hop; [P1] s5.3).
rr_algo_t pick_for(int n, size_t count, rr_dtype_t dtype, int align)
{
    if (n <= 1) return RR_ALGO_ONESHOT;
    rr_algo_t a = RR_ALGO_AUTO;
    if (!g_use_model.load(std::memory_order_relaxed)) a = table_pick(n, (uint64_t)count * esize(dtype), align);
    if (a == RR_ALGO_AUTO) a = model_pick(n, count, dtype);
    if (a == RR_ALGO_RING && (dtype == RR_BF16 || dtype == RR_F16)) a = RR_ALGO_ONESHOT;
    return a;
}

rr_algo_t resolve_algo(rr_algo_t algo, int n, size_t count, rr_dtype_t dtype, const void* const* bufs)
{
    if (algo != RR_ALGO_AUTO) return algo;
    static const int forced = [] {
        const char* v = std::getenv("RR_ALGO");
        if (!v) return -1;
        if (!std::strcmp(v, "ring")) return (int)RR_ALGO_RING;
        if (!std::strcmp(v, "oneshot")) return (int)RR_ALGO_ONESHOT;
        if (!std::strcmp(v, "tree")) return (int)RR_ALGO_TREE;
        if (!std::strcmp(v, "tree_oneshot")) return (int)RR_ALGO_TREE_ONESHOT;
        if (!std::strcmp(v, "two_shot")) return (int)RR_ALGO_TWO_SHOT;
        if (!std::strcmp(v, "double_ring")) return (int)RR_ALGO_DOUBLE_RING;
        return -1;
    }();
    if (forced >= 0) return (rr_algo_t)forced;
    return pick_for(n, count, dtype, bufs ? align_class(bufs, n) : 0);
}

// Slice size of the pipelined host-buffer all-reduce, per rank: 8 MiB, or
// RR_HOST_SLICE_MB (1..256) from the environment.
uint64_t host_slice_bytes()
{
    static const uint64_t v = [] {
        const char* e = std::getenv("RR_HOST_SLICE_MB");
        const long mb = e ? std::strtol(e, nullptr, 10) : 8;
        return (uint64_t)(mb >= 1 && mb <= 256 ? mb : 8) << 20;
    }();
    return v;
}

// Two copy streams and the events that order them against the caller's
// stream; created once per device and kept until exit.
struct HostPipe {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, arrived = nullptr, reduced = nullptr, done = nullptr;
};

rr_status_t host_pipe(HostPipe** out)
{
    static std::mutex mu;
    static std::unordered_map<int, HostPipe*> pipes;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    std::lock_guard<std::mutex> lock(mu);
    auto it = pipes.find(dev);
    if (it != pipes.end()) {
        *out = it->second;
        return RR_OK;
    }
    auto* hp = new HostPipe();
    const unsigned ef = cudaEventDisableTiming;
    if ((e = cudaStreamCreateWithFlags(&hp->in, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaStreamCreateWithFlags(&hp->out, cudaStreamNonBlocking)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp->start, ef)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp->arrived, ef)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp->reduced, ef)) != cudaSuccess ||
        (e = cudaEventCreateWithFlags(&hp->done, ef)) != cudaSuccess) {
        delete hp;
        return cuda_fail(e, "creating the copy streams");
    }
    pipes.emplace(dev, hp);
    *out = hp;
    return RR_OK;
}

}  // namespace

// Hooks for entry points defined in other files of the library: record the
// text rr_last_error() returns, and the statistics rr_get_stats() returns.
namespace rr {
rr_status_t record_error(rr_status_t st, const char* why)
{
    t_error = why;
    return st;
}

void record_stats(const rr_stats_t& s) { t_stats = s; }
}  // namespace rr

// ================================================================ C ABI ==

extern "C" {

int rr_version(void) { return RR_VERSION; }

rr_status_t rr_binary_version(int* version)
{
    if (!version) return fail(RR_ERR_INVALID_ARG, "NULL version pointer");
    const cudaError_t e = kernel_binary_version(version);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, "cudaFuncGetAttributes");
    }
    return RR_OK;
}

const char* rr_status_string(rr_status_t s)
{
    switch (s) {
    case RR_OK: return "ok";
    case RR_ERR_INVALID_ARG: return "invalid argument";
    case RR_ERR_UNSUPPORTED: return "unsupported";
    case RR_ERR_CUDA: return "CUDA error";
    case RR_ERR_TIMEOUT: return "timeout";
    }
    return "unknown status";
}

const char* rr_last_error(void) { return t_error.c_str(); }

rr_status_t rr_get_stats(rr_stats_t* out)
{
    if (!out) return fail(RR_ERR_INVALID_ARG, "NULL stats pointer");
    *out = t_stats;
    return RR_OK;
}

rr_status_t rr_allreduce(void* const* bufs, int nranks, size_t count, rr_dtype_t dtype, rr_op_t op,
                         rr_algo_t algo, cudaStream_t stream)
{
    CallTimer timer("rr_allreduce");
    rr_status_t st = check_basic(nranks, dtype, op);
    if (st != RR_OK) return st;
    if ((st = check_count(count)) != RR_OK) return st;
    if (algo < RR_ALGO_AUTO || algo > RR_ALGO_DOUBLE_RING) return fail(RR_ERR_INVALID_ARG, "unknown algo");
    if (!bufs) return fail(RR_ERR_INVALID_ARG, "NULL bufs array");
    const int n = nranks;
    const size_t es = esize(dtype);
    const rr_algo_t a = resolve_algo(algo, n, count, dtype, count && n <= RR_MAX_RANKS ? bufs : nullptr);
    stats_begin(a, n, (uint64_t)count * es);
    if (count == 0) return RR_OK;
    SpanBuf spans;
    for (int r = 0; r < n; ++r)
        spans.push_back({(uintptr_t)bufs[r], (uintptr_t)bufs[r] + count * es, true});
    if ((st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(bufs, n, es)) != RR_OK) return st;
    if ((st = check_device_ptrs(bufs, n)) != RR_OK) return st;
    if (n == 1) return RR_OK;  // one rank already holds the reduction (AVG: x / 1 == x)
    const uint64_t S = (uint64_t)count * es;
    switch (a) {
    case RR_ALGO_RING:
        st = run_ring(bufs, n, count, dtype, op, stream);
        break;
    case RR_ALGO_TREE:
        st = run_tree(bufs, n, count, dtype, op, stream);
        break;
    case RR_ALGO_DOUBLE_RING:
        st = run_double_ring(bufs, n, count, dtype, op, stream);
        break;
    case RR_ALGO_ONESHOT: {
        const uint64_t C = ceil_div(count, (uint64_t)n);
        const uint64_t tps = std::max<uint64_t>(1, ceil_div(C, tile_elems(dtype, reduce_vpt(n))));
        st = run_rank_kernel(kOneshotRing, bufs, bufs, n, C, count, (uint64_t)n, tps, dtype, op,
                             same_phase(bufs, n), stream);
        t_stats.steps = 1;
        t_stats.bytes_sent_max = (uint64_t)(n - 1) * S;  // each buffer is read by N-1 peers
        t_stats.bytes_sent_total = (uint64_t)n * (n - 1) * S;
        t_stats.hbm_bytes = 2ull * n * S;
        break;
    }
    case RR_ALGO_TWO_SHOT: {
        // shot 1: chunk c folded in ring order into rank c only; shot 2: every
        // rank copies the chunks it does not own from their owners
        const uint64_t C = ceil_div(count, (uint64_t)n);
        const bool vec = same_phase(bufs, n);
        uint64_t tps = std::max<uint64_t>(1, ceil_div(C, tile_elems(dtype, reduce_vpt(n))));
        st = run_rank_kernel(kOneshotRing, bufs, bufs, n, C, count, (uint64_t)n, tps, dtype, op, vec, stream, 0,
                             UINT64_MAX, true);
        if (st != RR_OK) break;
        tps = std::max<uint64_t>(1, ceil_div(C, tile_elems(dtype, kVptMove)));
        st = run_rank_kernel(kChunkBroadcast, bufs, bufs, n, C, count, (uint64_t)n, tps, dtype, RR_SUM, vec, stream);
        t_stats.steps = 2;
        t_stats.bytes_sent_max = 0;
        for (int r = 0; r < n; ++r) {  // r sends its copy of every other chunk, then its own chunk N-1 times
            const uint64_t own = chunk_len(count, n, r) * es;
            const uint64_t b = (S - own) + (uint64_t)(n - 1) * own;
            t_stats.bytes_sent_max = std::max(t_stats.bytes_sent_max, b);
            t_stats.bytes_sent_total += b;
        }
        t_stats.hbm_bytes = (2ull * n + 1) * S;  // shot 1: N S read, S written; shot 2: S read, (N-1) S written
        break;
    }
    case RR_ALGO_TREE_ONESHOT: {
        const uint64_t tps = std::max<uint64_t>(1, ceil_div(count, tile_elems(dtype, reduce_vpt(n))));
        st = run_rank_kernel(kOneshotTree, bufs, bufs, n, count, count, 1, tps, dtype, op, same_phase(bufs, n),
                             stream);
        t_stats.steps = 1;
        t_stats.bytes_sent_max = (uint64_t)(n - 1) * S;
        t_stats.bytes_sent_total = (uint64_t)n * (n - 1) * S;
        t_stats.hbm_bytes = 2ull * n * S;
        break;
    }
    default:
        return fail(RR_ERR_INVALID_ARG, "unknown algo");
    }
    log_call("allreduce", n, count, dtype, op, a);
    return debug_check(st, stream);
}

rr_status_t rr_allreduce_wire(void* const* bufs, int nranks, size_t count, rr_op_t op, rr_dtype_t wire,
                              rr_algo_t algo, cudaStream_t stream)
{
    CallTimer timer("rr_allreduce_wire");
    rr_status_t st = check_basic(nranks, RR_F32, op);
    if (st != RR_OK) return st;
    if ((st = check_count(count)) != RR_OK) return st;
    if (op != RR_SUM && op != RR_AVG) return fail(RR_ERR_UNSUPPORTED, "the wire format carries SUM or AVG");
    if (wire != RR_BF16) return fail(RR_ERR_UNSUPPORTED, "the wire format is bf16");
    if (algo != RR_ALGO_AUTO && algo != RR_ALGO_ONESHOT && algo != RR_ALGO_RING)
        return fail(RR_ERR_UNSUPPORTED, "the bf16 wire runs AUTO, ONESHOT or RING");
    if (!bufs) return fail(RR_ERR_INVALID_ARG, "NULL bufs array");
    const int n = nranks;
    const rr_algo_t a = algo == RR_ALGO_RING ? RR_ALGO_RING : RR_ALGO_ONESHOT;
    const uint64_t S = (uint64_t)count * 4;
    stats_begin(a, n, S);
    if (count == 0) return RR_OK;
    SpanBuf spans;
    for (int r = 0; r < n; ++r) spans.push_back({(uintptr_t)bufs[r], (uintptr_t)bufs[r] + S, true});
    if ((st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(bufs, n, 4)) != RR_OK) return st;
    if ((st = check_device_ptrs(bufs, n)) != RR_OK) return st;
    if (n == 1) return RR_OK;  // nothing crosses a wire
    if (a == RR_ALGO_RING) {
        if ((st = run_ring(bufs, n, count, RR_F32, op, stream, true)) != RR_OK) return st;
    } else {
        RankParams p{};
        for (int r = 0; r < n; ++r) p.in[r] = p.out[r] = bufs[r];
        p.n = n;
        p.vec_ok = same_phase(bufs, n);
        p.divisor = (float)n;
        p.C = ceil_div(count, (uint64_t)n);
        p.count = count;
        p.nseg = (uint64_t)n;
        p.tps = std::max<uint64_t>(1, ceil_div(p.C, tile_elems(RR_F32, kVptReduce)));
        p.lo = 0;
        p.hi = UINT64_MAX;
        p.waits = bulk_wait_counters();
        cudaError_t e = timed_launch([&] { return launch_oneshot_wire(op, p, p.nseg * p.tps, stream); });
        if (e != cudaSuccess) return cuda_fail(e, "wire one-shot launch");
        t_stats.launches = 1;
        t_stats.steps = 1;
        t_stats.bytes_sent_max = (uint64_t)(n - 1) * count * 2;  // each rank's values go out as bf16
        t_stats.bytes_sent_total = (uint64_t)n * t_stats.bytes_sent_max;
        t_stats.hbm_bytes = 2ull * n * S;
    }
    log_call("allreduce_wire", n, count, RR_F32, op, a);
    return debug_check(RR_OK, stream);
}

rr_status_t rr_allreduce_host(void* const* host_bufs, void* const* dev_bufs, int nranks, size_t count,
                              rr_dtype_t dtype, rr_op_t op, rr_algo_t algo, cudaStream_t stream)
{
    CallTimer timer("rr_allreduce_host");
    rr_status_t st = check_basic(nranks, dtype, op);
    if (st != RR_OK) return st;
    if ((st = check_count(count)) != RR_OK) return st;
    if (algo < RR_ALGO_AUTO || algo > RR_ALGO_DOUBLE_RING) return fail(RR_ERR_INVALID_ARG, "unknown algo");
    if (!host_bufs || !dev_bufs) return fail(RR_ERR_INVALID_ARG, "NULL pointer array");
    const int n = nranks;
    const size_t es = esize(dtype), bytes = count * es;
    for (int r = 0; r < n && count; ++r)
        if (!host_bufs[r]) return fail(RR_ERR_INVALID_ARG, "NULL host buffer");
    SpanBuf spans;  // host buffers are written back too (one address space with UVA)
    for (int r = 0; r < n && count; ++r) {
        spans.push_back({(uintptr_t)dev_bufs[r], (uintptr_t)dev_bufs[r] + bytes, true});
        spans.push_back({(uintptr_t)host_bufs[r], (uintptr_t)host_bufs[r] + bytes, true});
    }
    if ((st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(dev_bufs, n, es)) != RR_OK) return st;
    const rr_algo_t a = resolve_algo(algo, n, count, dtype, count ? dev_bufs : nullptr);
    if (count == 0) return rr_allreduce(dev_bufs, n, 0, dtype, op, a, stream);
    const bool sliced = n > 1 && (a == RR_ALGO_ONESHOT || a == RR_ALGO_TREE_ONESHOT) && bytes > host_slice_bytes();
    if (!sliced) {  // copy in, reduce, copy out, all on the caller's stream
        for (int r = 0; r < n; ++r) {
            cudaError_t e = cudaMemcpyAsync(dev_bufs[r], host_bufs[r], bytes, cudaMemcpyHostToDevice, stream);
            if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
        }
        if ((st = rr_allreduce(dev_bufs, n, count, dtype, op, a, stream)) != RR_OK) return st;
        for (int r = 0; r < n; ++r) {
            cudaError_t e = cudaMemcpyAsync(host_bufs[r], dev_bufs[r], bytes, cudaMemcpyDeviceToHost, stream);
            if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
        }
        return RR_OK;
    }
    // Pipelined: slice k of every rank is uploaded on one stream, reduced on
    // the caller's stream once it has arrived, and downloaded on another
    // stream, so uploads and downloads of different slices overlap.  The
    // one-shot fold is element-local, so each slice reduces on its own with
    // the chunk rule of the whole buffer.
    HostPipe* hp = nullptr;
    if ((st = host_pipe(&hp)) != RR_OK) return st;
    auto ck = [&](cudaError_t e, const char* where) { return e == cudaSuccess ? RR_OK : cuda_fail(e, where); };
    if ((st = ck(cudaEventRecord(hp->start, stream), "event record")) != RR_OK) return st;
    if ((st = ck(cudaStreamWaitEvent(hp->in, hp->start, 0), "stream wait")) != RR_OK) return st;
    if ((st = ck(cudaStreamWaitEvent(hp->out, hp->start, 0), "stream wait")) != RR_OK) return st;
    const uint64_t slice = std::max<uint64_t>(1, host_slice_bytes() / es);
    const uint64_t C = ceil_div(count, (uint64_t)n);
    const bool vec = same_phase(dev_bufs, n);
    int launches = 0;
    for (uint64_t lo = 0; lo < count; lo += slice) {
        const uint64_t hi = std::min<uint64_t>(count, lo + slice), len = hi - lo;
        for (int r = 0; r < n; ++r) {
            cudaError_t e = cudaMemcpyAsync(static_cast<char*>(dev_bufs[r]) + lo * es,
                                            static_cast<const char*>(host_bufs[r]) + lo * es, len * es,
                                            cudaMemcpyHostToDevice, hp->in);
            if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
        }
        if ((st = ck(cudaEventRecord(hp->arrived, hp->in), "event record")) != RR_OK) return st;
        if ((st = ck(cudaStreamWaitEvent(stream, hp->arrived, 0), "stream wait")) != RR_OK) return st;
        if (a == RR_ALGO_ONESHOT) {
            const uint64_t tps =
                std::max<uint64_t>(1, ceil_div(std::min(C, len), tile_elems(dtype, reduce_vpt(n))));
            st = run_rank_kernel(kOneshotRing, dev_bufs, dev_bufs, n, C, count, (uint64_t)n, tps, dtype, op, vec,
                                 stream, lo, hi);
        } else {
            void* off[RR_MAX_RANKS];
            for (int r = 0; r < n; ++r) off[r] = static_cast<char*>(dev_bufs[r]) + lo * es;
            const uint64_t tps = std::max<uint64_t>(1, ceil_div(len, tile_elems(dtype, reduce_vpt(n))));
            st = run_rank_kernel(kOneshotTree, off, off, n, len, len, 1, tps, dtype, op, same_phase(off, n), stream);
        }
        if (st != RR_OK) return st;
        ++launches;
        if ((st = ck(cudaEventRecord(hp->reduced, stream), "event record")) != RR_OK) return st;
        if ((st = ck(cudaStreamWaitEvent(hp->out, hp->reduced, 0), "stream wait")) != RR_OK) return st;
        for (int r = 0; r < n; ++r) {
            cudaError_t e = cudaMemcpyAsync(static_cast<char*>(host_bufs[r]) + lo * es,
                                            static_cast<const char*>(dev_bufs[r]) + lo * es, len * es,
                                            cudaMemcpyDeviceToHost, hp->out);
            if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
        }
    }
    if ((st = ck(cudaEventRecord(hp->done, hp->out), "event record")) != RR_OK) return st;
    if ((st = ck(cudaStreamWaitEvent(stream, hp->done, 0), "stream wait")) != RR_OK) return st;
    const uint64_t launch_ns = t_stats.launch_ns;
    stats_begin(a, n, bytes);
    t_stats.launch_ns = launch_ns;
    t_stats.steps = 1;
    t_stats.launches = launches;
    t_stats.bytes_sent_max = (uint64_t)(n - 1) * bytes;
    t_stats.bytes_sent_total = (uint64_t)n * (n - 1) * bytes;
    t_stats.hbm_bytes = 4ull * n * bytes;  // copies in and out, plus the fold's read and write
    log_call("allreduce_host", n, count, dtype, op, a);
    return RR_OK;
}

rr_status_t rr_ring_step(void* const* bufs, int nranks, size_t count, rr_dtype_t dtype, rr_op_t op,
                         rr_phase_t phase, int step, cudaStream_t stream)
{
    CallTimer timer("rr_ring_step");
    rr_status_t st = check_basic(nranks, dtype, op);
    if (st != RR_OK) return st;
    if ((st = check_count(count)) != RR_OK) return st;
    if (phase != RR_PHASE_REDUCE_SCATTER && phase != RR_PHASE_ALL_GATHER)
        return fail(RR_ERR_INVALID_ARG, "unknown phase");
    if (step < 0 || step > nranks - 2) return fail(RR_ERR_INVALID_ARG, "step must be in 0..nranks-2");
    if (!bufs) return fail(RR_ERR_INVALID_ARG, "NULL bufs array");
    const size_t es = esize(dtype);
    stats_begin(RR_ALGO_RING, nranks, (uint64_t)count * es);
    if (count == 0) return RR_OK;
    SpanBuf spans;
    for (int r = 0; r < nranks; ++r)
        spans.push_back({(uintptr_t)bufs[r], (uintptr_t)bufs[r] + count * es, true});
    if ((st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(bufs, nranks, es)) != RR_OK) return st;
    if ((st = check_device_ptrs(bufs, nranks)) != RR_OK) return st;
    st = ring_step_launch(bufs, nranks, count, dtype, op, phase, step, stream);
    t_stats.steps = 1;
    for (int r = 0; r < nranks; ++r) {
        const uint64_t b = chunk_len(count, nranks, ring_send_chunk(phase, r, step, nranks)) * es;
        t_stats.bytes_sent_max = std::max(t_stats.bytes_sent_max, b);
        t_stats.bytes_sent_total += b;
    }
    t_stats.hbm_bytes = (phase == RR_PHASE_REDUCE_SCATTER ? 3ull : 2ull) * count * es;
    log_call("ring_step", nranks, count, dtype, op, RR_ALGO_RING);
    return debug_check(st, stream);
}

rr_status_t rr_ring_schedule(int nranks, size_t count, rr_dtype_t dtype, rr_ring_event_t* events,
                             size_t capacity, size_t* nevents)
{
    if (nranks < 1 || nranks > RR_MAX_RANKS) return fail(RR_ERR_INVALID_ARG, "nranks must be in 1..64");
    if (!dtype_ok(dtype)) return fail(RR_ERR_INVALID_ARG, "unknown dtype");
    const int n = nranks;
    const size_t total = 2ull * (size_t)(n - 1) * (size_t)n;
    if (nevents) *nevents = total;
    if (total > capacity || (total && !events)) return fail(RR_ERR_INVALID_ARG, "events capacity too small");
    size_t i = 0;
    for (int phase = RR_PHASE_REDUCE_SCATTER; phase <= RR_PHASE_ALL_GATHER; ++phase)
        for (int s = 0; s < n - 1; ++s)
            for (int r = 0; r < n; ++r) {
                rr_ring_event_t& e = events[i++];
                e.phase = phase;
                e.step = s;
                e.rank = r;
                e.dst = imod(r + 1, n);
                e.send_idx = ring_send_chunk(phase, r, s, n);
                e.recv_idx = ring_send_chunk(phase, imod(r - 1, n), s, n);
                e.bytes = chunk_len(count, n, e.send_idx) * esize(dtype);
            }
    return RR_OK;
}

rr_status_t rr_reduce_scatter(const void* const* send, void* const* recv, int nranks, size_t recvcount,
                              rr_dtype_t dtype, rr_op_t op, rr_algo_t algo, cudaStream_t stream)
{
    CallTimer timer("rr_reduce_scatter");
    rr_status_t st = check_basic(nranks, dtype, op);
    if (st != RR_OK) return st;
    if ((st = check_count(recvcount)) != RR_OK) return st;
    if (algo != RR_ALGO_AUTO && algo != RR_ALGO_ONESHOT)
        return fail(RR_ERR_UNSUPPORTED, "reduce-scatter runs AUTO or ONESHOT");
    if (!send || !recv) return fail(RR_ERR_INVALID_ARG, "NULL pointer array");
    const int n = nranks;
    const size_t es = esize(dtype);
    const uint64_t S = (uint64_t)n * recvcount * es;
    stats_begin(RR_ALGO_ONESHOT, n, S);
    if (recvcount == 0) return RR_OK;
    SpanBuf spans;
    for (int r = 0; r < n; ++r) {
        spans.push_back({(uintptr_t)send[r], (uintptr_t)send[r] + S, false});
        spans.push_back({(uintptr_t)recv[r], (uintptr_t)recv[r] + recvcount * es, true});
    }
    if ((st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(send, n, es)) != RR_OK || (st = check_elem_aligned(recv, n, es)) != RR_OK) return st;
    if ((st = check_device_ptrs(send, n)) != RR_OK || (st = check_device_ptrs(recv, n)) != RR_OK) return st;
    const uint64_t tps = std::max<uint64_t>(1, ceil_div(recvcount, tile_elems(dtype, reduce_vpt(n))));
    st = run_rank_kernel(kReduceScatter, send, recv, n, recvcount, (uint64_t)n * recvcount, (uint64_t)n, tps,
                         dtype, op, same_phase(send, n) && same_phase(recv, n), stream);
    t_stats.steps = 1;
    t_stats.bytes_sent_max = (uint64_t)(n - 1) * recvcount * es;  // (N-1)/N S ([P4])
    t_stats.bytes_sent_total = (uint64_t)n * t_stats.bytes_sent_max;
    t_stats.hbm_bytes = (uint64_t)(n + 1) * S;
    log_call("reduce_scatter", n, recvcount, dtype, op, RR_ALGO_ONESHOT);
    return debug_check(st, stream);
}

rr_status_t rr_all_gather(const void* const* send, void* const* recv, int nranks, size_t sendcount,
                          rr_dtype_t dtype, rr_algo_t algo, cudaStream_t stream)
{
    CallTimer timer("rr_all_gather");
    rr_status_t st = check_basic(nranks, dtype, RR_SUM);
    if (st != RR_OK) return st;
    if ((st = check_count(sendcount)) != RR_OK) return st;
    if (algo != RR_ALGO_AUTO && algo != RR_ALGO_ONESHOT)
        return fail(RR_ERR_UNSUPPORTED, "all-gather runs AUTO or ONESHOT");
    if (!send || !recv) return fail(RR_ERR_INVALID_ARG, "NULL pointer array");
    const int n = nranks;
    const size_t es = esize(dtype);
    const uint64_t S = (uint64_t)n * sendcount * es;
    stats_begin(RR_ALGO_ONESHOT, n, S);
    if (sendcount == 0) return RR_OK;
    SpanBuf spans;
    for (int r = 0; r < n; ++r) {
        spans.push_back({(uintptr_t)send[r], (uintptr_t)send[r] + sendcount * es, false});
        spans.push_back({(uintptr_t)recv[r], (uintptr_t)recv[r] + S, true});
    }
    if ((st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(send, n, es)) != RR_OK || (st = check_elem_aligned(recv, n, es)) != RR_OK) return st;
    if ((st = check_device_ptrs(send, n)) != RR_OK || (st = check_device_ptrs(recv, n)) != RR_OK) return st;
    const uint64_t tps = std::max<uint64_t>(1, ceil_div(sendcount, tile_elems(dtype, kVptMove)));
    st = run_rank_kernel(kAllGather, send, recv, n, sendcount, (uint64_t)n * sendcount, (uint64_t)n, tps, dtype,
                         RR_SUM, same_phase(send, n) && same_phase(recv, n), stream);
    t_stats.steps = 1;
    t_stats.bytes_sent_max = (uint64_t)(n - 1) * sendcount * es;
    t_stats.bytes_sent_total = (uint64_t)n * t_stats.bytes_sent_max;
    t_stats.hbm_bytes = (uint64_t)(n + 1) * S;
    log_call("all_gather", n, sendcount, dtype, RR_SUM, RR_ALGO_ONESHOT);
    return debug_check(st, stream);
}

rr_status_t rr_all_to_all(const void* const* send, void* const* recv, int nranks, size_t count_per_peer,
                          rr_dtype_t dtype, cudaStream_t stream)
{
    CallTimer timer("rr_all_to_all");
    rr_status_t st = check_basic(nranks, dtype, RR_SUM);
    if (st != RR_OK) return st;
    if ((st = check_count(count_per_peer)) != RR_OK) return st;
    if (!send || !recv) return fail(RR_ERR_INVALID_ARG, "NULL pointer array");
    const int n = nranks;
    const size_t es = esize(dtype);
    const uint64_t S = (uint64_t)n * count_per_peer * es;
    stats_begin(RR_ALGO_ONESHOT, n, S);
    if (count_per_peer == 0) return RR_OK;
    SpanBuf spans;
    for (int r = 0; r < n; ++r) {
        spans.push_back({(uintptr_t)send[r], (uintptr_t)send[r] + S, false});
        spans.push_back({(uintptr_t)recv[r], (uintptr_t)recv[r] + S, true});
    }
    if ((st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(send, n, es)) != RR_OK || (st = check_elem_aligned(recv, n, es)) != RR_OK) return st;
    if ((st = check_device_ptrs(send, n)) != RR_OK || (st = check_device_ptrs(recv, n)) != RR_OK) return st;
    const uint64_t tps = std::max<uint64_t>(1, ceil_div(count_per_peer, tile_elems(dtype, kVptMove)));
    st = run_rank_kernel(kAllToAll, send, recv, n, count_per_peer, (uint64_t)n * count_per_peer,
                         (uint64_t)n * n, tps, dtype, RR_SUM, true, stream);
    t_stats.steps = 1;
    t_stats.bytes_sent_max = (uint64_t)(n - 1) * count_per_peer * es;  // own block stays ([P4])
    t_stats.bytes_sent_total = (uint64_t)n * t_stats.bytes_sent_max;
    t_stats.hbm_bytes = 2ull * n * S;
    log_call("all_to_all", n, count_per_peer, dtype, RR_SUM, RR_ALGO_ONESHOT);
    return debug_check(st, stream);
}

// ------------------------------------------------------------- buckets --

rr_status_t rr_bucket_plan(const size_t* numels, int ntensors, rr_dtype_t grad_dtype, size_t cap_bytes,
                           rr_bucket_plan_t** out)
{
    if (!out) return fail(RR_ERR_INVALID_ARG, "NULL plan output");
    *out = nullptr;
    if (ntensors < 0 || (ntensors > 0 && !numels)) return fail(RR_ERR_INVALID_ARG, "bad tensor list");
    if (grad_dtype != RR_BF16 && grad_dtype != RR_F16 && grad_dtype != RR_F32)
        return fail(RR_ERR_UNSUPPORTED, "gradients must be bf16, fp16 or fp32");
    auto* p = new rr_bucket_plan_t();
    p->ntensors = ntensors;
    p->grad_dtype = grad_dtype;
    p->cap_bytes = cap_bytes;
    const uint64_t es = esize(grad_dtype);
    uint64_t off = 0, bytes = 0;
    int b = 0, open = 0;
    for (int t = 0; t < ntensors; ++t) {
        if (numels[t] > kMaxElems || off + numels[t] > kMaxElems) {
            delete p;
            return fail(RR_ERR_INVALID_ARG, "element count above 2^48");
        }
        if (!open) {
            p->first.push_back(t);
            p->count.push_back(0);
            p->bnumel.push_back(0);
            open = 1;
        }
        p->numel.push_back(numels[t]);
        p->offset.push_back(off);
        p->bucket_of.push_back(b);
        p->count[b] += 1;
        off += numels[t];
        p->bnumel[b] = off;
        bytes += numels[t] * es;
        if (bytes >= cap_bytes) {  // the bucket reached the cap: close it
            ++b;
            off = 0;
            bytes = 0;
            open = 0;
        }
    }
    *out = p;
    return RR_OK;
}

void rr_bucket_plan_free(rr_bucket_plan_t* plan) { delete plan; }

int rr_bucket_count(const rr_bucket_plan_t* plan) { return plan ? (int)plan->first.size() : 0; }

rr_status_t rr_bucket_info(const rr_bucket_plan_t* plan, int bucket, int* first_tensor, int* ntensors,
                           size_t* numel)
{
    if (!plan || bucket < 0 || bucket >= (int)plan->first.size()) return fail(RR_ERR_INVALID_ARG, "bad bucket");
    if (first_tensor) *first_tensor = plan->first[bucket];
    if (ntensors) *ntensors = plan->count[bucket];
    if (numel) *numel = plan->bnumel[bucket];
    return RR_OK;
}

rr_status_t rr_bucket_tensor(const rr_bucket_plan_t* plan, int tensor, int* bucket, size_t* offset)
{
    if (!plan || tensor < 0 || tensor >= plan->ntensors) return fail(RR_ERR_INVALID_ARG, "bad tensor");
    if (bucket) *bucket = plan->bucket_of[tensor];
    if (offset) *offset = plan->offset[tensor];
    return RR_OK;
}

namespace {

// Checks shared by the bucket calls; fills the bucket's tensor range.
// Checks buckets [b0, b0 + nb) of a plan and the gradients they cover (every
// rank's copy of every tensor in the range, pairwise disjoint); *t0 and *nt
// are the range's first tensor and tensor count.
rr_status_t bucket_range_check(const rr_bucket_plan_t* plan, int b0, int nb, const void* const* grads, int nranks,
                               int* t0, int* nt)
{
    if (!plan) return fail(RR_ERR_INVALID_ARG, "NULL plan");
    if (nranks < 1 || nranks > RR_MAX_RANKS) return fail(RR_ERR_INVALID_ARG, "nranks must be in 1..64");
    const int nbk = (int)plan->first.size();
    if (b0 < 0 || nb < 1 || b0 >= nbk || nb > nbk - b0) return fail(RR_ERR_INVALID_ARG, "bad bucket");
    if (!grads) return fail(RR_ERR_INVALID_ARG, "NULL gradient array");
    *t0 = plan->first[b0];
    *nt = plan->first[b0 + nb - 1] + plan->count[b0 + nb - 1] - *t0;
    const uint64_t es = esize((rr_dtype_t)plan->grad_dtype);
    std::vector<Span> spans;
    for (int r = 0; r < nranks; ++r)
        for (int t = *t0; t < *t0 + *nt; ++t) {
            const void* g = grads[(size_t)r * plan->ntensors + t];
            if (plan->numel[t] == 0) continue;
            if ((uintptr_t)g % es != 0) return fail(RR_ERR_INVALID_ARG, "gradient not aligned to its element size");
            spans.push_back({(uintptr_t)g, (uintptr_t)g + plan->numel[t] * es, true});
        }
    return check_spans(spans);
}

rr_status_t bucket_check(const rr_bucket_plan_t* plan, int bucket, const void* const* grads, int nranks, int* t0,
                         int* nt)
{
    return bucket_range_check(plan, bucket, 1, grads, nranks, t0, nt);
}

}  // namespace

static rr_status_t bucket_copy(const rr_bucket_plan_t* plan, int bucket, const void* const* grads,
                               void* const* buckets, int nranks, int op, bool pack, cudaStream_t stream)
{
    CallTimer timer(pack ? "rr_bucket_pack" : "rr_bucket_unpack");
    int t0 = 0, nt = 0;
    rr_status_t st = bucket_check(plan, bucket, grads, nranks, &t0, &nt);
    if (st != RR_OK) return st;
    if (!buckets) return fail(RR_ERR_INVALID_ARG, "NULL bucket array");
    const int n = nranks;
    const uint64_t es = esize((rr_dtype_t)plan->grad_dtype);
    stats_begin(RR_ALGO_ONESHOT, n, plan->bnumel[bucket] * 4);
    std::vector<Span> spans;
    for (int r = 0; r < n; ++r)
        spans.push_back({(uintptr_t)buckets[r], (uintptr_t)buckets[r] + plan->bnumel[bucket] * 4, true});
    if (plan->bnumel[bucket] && (st = check_spans(spans)) != RR_OK) return st;
    if ((st = check_elem_aligned(buckets, n, 4)) != RR_OK) return st;
    const int per_launch = std::max(1, std::min(kMaxBucketTensors, kMaxBucketPtrs / n));
    auto* p = new BucketCopyParams();
    for (int g0 = 0; g0 < nt; g0 += per_launch) {
        const int g1 = std::min(nt, g0 + per_launch);
        *p = BucketCopyParams{};
        p->n = n;
        p->nt = g1 - g0;
        p->divisor = (float)n;
        uint64_t maxlen = 0;
        const uint64_t te = bucket_tile_elems(plan->grad_dtype);
        p->tile0[0] = 0;
        for (int t = g0; t < g1; ++t) {
            const int gt = t0 + t;
            for (int r = 0; r < n; ++r) p->grad[(t - g0) * n + r] = grads[(size_t)r * plan->ntensors + gt];
            p->toff[t - g0] = plan->offset[gt];
            p->tlen[t - g0] = plan->numel[gt];
            p->tile0[t - g0 + 1] = p->tile0[t - g0] + (uint64_t)n * ceil_div(plan->numel[gt], te);
            maxlen = std::max<uint64_t>(maxlen, plan->numel[gt]);
        }
        for (int r = 0; r < n; ++r) p->bucket[r] = buckets[r];
        if (maxlen == 0) continue;
        cudaError_t e = timed_launch([&] {
            return pack ? launch_bucket_pack(plan->grad_dtype, *p, stream)
                        : launch_bucket_unpack(plan->grad_dtype, op, *p, stream);
        });
        if (e != cudaSuccess) {
            delete p;
            return cuda_fail(e, pack ? "bucket pack launch" : "bucket unpack launch");
        }
        t_stats.launches += 1;
    }
    delete p;
    t_stats.steps = 1;
    t_stats.hbm_bytes = (uint64_t)n * plan->bnumel[bucket] * (es + 4);
    return RR_OK;
}

rr_status_t rr_bucket_pack(const rr_bucket_plan_t* plan, int bucket, const void* const* grads,
                           void* const* buckets, int nranks, cudaStream_t stream)
{
    rr_status_t st = bucket_copy(plan, bucket, grads, buckets, nranks, RR_SUM, true, stream);
    log_call("bucket_pack", nranks, plan ? (size_t)plan->bnumel[std::max(0, bucket)] : 0, RR_F32, RR_SUM,
             RR_ALGO_ONESHOT);
    return st;
}

rr_status_t rr_bucket_unpack(const rr_bucket_plan_t* plan, int bucket, const void* const* buckets,
                             void* const* grads, int nranks, rr_op_t op, cudaStream_t stream)
{
    if (op != RR_SUM && op != RR_AVG) return fail(RR_ERR_UNSUPPORTED, "bucket unpack takes SUM or AVG");
    return bucket_copy(plan, bucket, grads, const_cast<void* const*>(buckets), nranks, op, false, stream);
}

static rr_status_t bucket_fold_range(const rr_bucket_plan_t* plan, int b0, int nb, void* const* grads, int nranks,
                                     rr_op_t op, cudaStream_t stream, uint64_t max_grid, bool pdl);

rr_status_t rr_bucket_allreduce(const rr_bucket_plan_t* plan, int bucket, void* const* grads, int nranks,
                                rr_op_t op, cudaStream_t stream)
{
    return bucket_fold_range(plan, bucket, 1, grads, nranks, op, stream, kMaxGrid, true);
}

rr_status_t rr_bucket_allreduce_range(const rr_bucket_plan_t* plan, int first_bucket, int nbuckets, void* const* grads,
                                      int nranks, rr_op_t op, cudaStream_t stream)
{
    return bucket_fold_range(plan, first_bucket, nbuckets, grads, nranks, op, stream, kMaxGrid, true);
}

}  // extern "C"

// The fused sync of buckets [b0, b0 + nb): every bucket is chunked over its
// own flat index (chunk size ceil(bucket numel / N)) exactly as a sync of
// that bucket alone, and its tensors are split at its chunk boundaries into
// segments (tensor, chunk); segments of consecutive buckets share a launch
// until the parameter block is full, so a range costs a few launches instead
// of one per bucket, with the same bits.
static rr_status_t bucket_fold_range(const rr_bucket_plan_t* plan, int b0, int nb, void* const* grads, int nranks,
                                     rr_op_t op, cudaStream_t stream, uint64_t max_grid, bool pdl)
{
    CallTimer timer("rr_bucket_allreduce");
    if (op != RR_SUM && op != RR_AVG) return fail(RR_ERR_UNSUPPORTED, "bucket all-reduce takes SUM or AVG");
    int t0 = 0, nt = 0;
    rr_status_t st = bucket_range_check(plan, b0, nb, grads, nranks, &t0, &nt);
    if (st != RR_OK) return st;
    const int n = nranks;
    const uint64_t es = esize((rr_dtype_t)plan->grad_dtype);
    uint64_t total = 0;
    for (int b = b0; b < b0 + nb; ++b) total += plan->bnumel[b];
    stats_begin(RR_ALGO_ONESHOT, n, total * es);
    if (n == 1 || total == 0) return RR_OK;
    auto* p = new BucketFoldParams();
    auto flush = [&](int ntens) -> rr_status_t {
        if (p->nseg == 0) return RR_OK;
        const uint64_t te = tile_elems(plan->grad_dtype, reduce_vpt(n));
        p->tile0[0] = 0;
        for (int s = 0; s < p->nseg; ++s) p->tile0[s + 1] = p->tile0[s] + ceil_div(p->seg[s].len, te);
        p->n = n;
        p->divisor = (float)n;
        bool v = true;
        for (int t = 0; t < ntens; ++t) v = v && same_phase(&p->grad[t * n], n);
        p->vec_ok = v;
        cudaError_t e =
            timed_launch([&] { return launch_bucket_fold(plan->grad_dtype, op, *p, stream, max_grid, pdl); });
        if (e != cudaSuccess) return cuda_fail(e, "bucket all-reduce launch");
        t_stats.launches += 1;
        return RR_OK;
    };
    int lt = 0;  // tensors in the current launch
    *p = BucketFoldParams{};
    for (int b = b0; b < b0 + nb && st == RR_OK; ++b) {
        const uint64_t C = ceil_div(plan->bnumel[b], (uint64_t)n);  // this bucket's chunk size
        for (int t = plan->first[b]; t < plan->first[b] + plan->count[b] && st == RR_OK; ++t) {
            const uint64_t lo = plan->offset[t], hi = lo + plan->numel[t];  // offsets are bucket-relative
            const int nsegs_t = hi > lo ? (int)((hi - 1) / C - lo / C + 1) : 0;
            if (lt + 1 > kMaxBucketTensors || (lt + 1) * n > kMaxBucketPtrs || p->nseg + nsegs_t > kMaxBucketSegs) {
                st = flush(lt);
                *p = BucketFoldParams{};
                lt = 0;
            }
            for (int r = 0; r < n; ++r) p->grad[lt * n + r] = grads[(size_t)r * plan->ntensors + t];
            for (uint64_t pos = lo; pos < hi;) {  // split the tensor at the bucket's chunk boundaries
                const uint64_t c = pos / C, end = std::min(hi, (c + 1) * C);
                p->seg[p->nseg++] = BucketSeg{(uint32_t)lt, (uint32_t)c, pos - lo, end - pos};
                pos = end;
            }
            ++lt;
        }
    }
    if (st == RR_OK) st = flush(lt);
    delete p;
    t_stats.steps = 1;
    t_stats.bytes_sent_max = (uint64_t)(n - 1) * total * es;
    t_stats.bytes_sent_total = (uint64_t)n * t_stats.bytes_sent_max;
    t_stats.hbm_bytes = 2ull * n * total * es;
    log_call("bucket_allreduce", n, total, (rr_dtype_t)plan->grad_dtype, op, RR_ALGO_ONESHOT);
    return debug_check(st, stream);
}

extern "C" {

// -------------------------------------------------------------- reducer --

}  // extern "C"

struct rr_reducer {
    const rr_bucket_plan_t* plan = nullptr;
    int n = 0;
    rr_op_t op = RR_AVG;
    cudaStream_t comm = nullptr;
    uint64_t max_grid = kMaxGrid;     // CTAs of each bucket sync
    std::vector<void*> grads;         // nranks * ntensors, rank-major
    std::vector<int> pending;         // per bucket: tensors not yet marked in this step
    std::vector<char> marked;         // per tensor
    std::vector<cudaEvent_t> ready;   // per bucket: recorded on the producer when it completes
    cudaEvent_t done = nullptr;       // recorded on comm at the end of a step

    void reset()
    {
        for (size_t b = 0; b < pending.size(); ++b) pending[b] = plan->count[b];
        std::fill(marked.begin(), marked.end(), 0);
    }
    ~rr_reducer()
    {
        for (cudaEvent_t e : ready)
            if (e) cudaEventDestroy(e);
        if (done) cudaEventDestroy(done);
    }
};

extern "C" {

rr_status_t rr_reducer_create(const rr_bucket_plan_t* plan, void* const* grads, int nranks, rr_op_t op,
                              cudaStream_t comm, int max_ctas, rr_reducer_t** out)
{
    if (!out) return fail(RR_ERR_INVALID_ARG, "NULL reducer output");
    *out = nullptr;
    if (!plan || !grads) return fail(RR_ERR_INVALID_ARG, "NULL plan or gradient array");
    if (nranks < 1 || nranks > RR_MAX_RANKS) return fail(RR_ERR_INVALID_ARG, "nranks must be in 1..64");
    if (op != RR_SUM && op != RR_AVG) return fail(RR_ERR_UNSUPPORTED, "the reducer takes SUM or AVG");
    if (!plan->first.empty()) {  // every gradient of every bucket, once, before any step
        int t0 = 0, nt = 0;
        rr_status_t st = bucket_range_check(plan, 0, (int)plan->first.size(), grads, nranks, &t0, &nt);
        if (st != RR_OK) return st;
    }
    auto* red = new rr_reducer();
    red->plan = plan;
    red->n = nranks;
    red->op = op;
    red->comm = comm;
    red->max_grid = max_ctas > 0 ? (uint64_t)max_ctas : kMaxGrid;
    red->grads.assign(grads, grads + (size_t)nranks * plan->ntensors);
    const int nb = (int)plan->first.size();
    red->pending.assign(nb, 0);
    red->marked.assign(plan->ntensors, 0);
    red->ready.assign(nb, nullptr);
    for (int b = 0; b < nb; ++b) {
        cudaError_t e = cudaEventCreateWithFlags(&red->ready[b], cudaEventDisableTiming);
        if (e != cudaSuccess) {
            delete red;
            return cuda_fail(e, "creating the reducer's events");
        }
    }
    cudaError_t e = cudaEventCreateWithFlags(&red->done, cudaEventDisableTiming);
    if (e != cudaSuccess) {
        delete red;
        return cuda_fail(e, "creating the reducer's events");
    }
    red->reset();
    *out = red;
    return RR_OK;
}

rr_status_t rr_reducer_ready(rr_reducer_t* red, int tensor, cudaStream_t producer)
{
    if (!red) return fail(RR_ERR_INVALID_ARG, "NULL reducer");
    if (tensor < 0 || tensor >= red->plan->ntensors) return fail(RR_ERR_INVALID_ARG, "bad tensor");
    if (red->marked[tensor]) return fail(RR_ERR_INVALID_ARG, "tensor marked ready twice in one step");
    red->marked[tensor] = 1;
    const int b = red->plan->bucket_of[tensor];
    if (--red->pending[b] > 0) return RR_OK;
    cudaError_t e = cudaEventRecord(red->ready[b], producer);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(red->comm, red->ready[b], 0);
    if (e != cudaSuccess) return cuda_fail(e, "ordering the bucket sync after its gradients");
    return bucket_fold_range(red->plan, b, 1, red->grads.data(), red->n, red->op, red->comm, red->max_grid, false);
}

rr_status_t rr_check_timeouts(void)
{
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "synchronising before reading the wait counters");
    unsigned int ran_out = 0, in_flight = 0;
    if ((e = take_bulk_timeouts(&ran_out, &in_flight)) != cudaSuccess) return cuda_fail(e, "reading the wait counters");
    if (ran_out || in_flight)
        return fail(RR_ERR_TIMEOUT, "bounded device waits ran out on " + std::to_string(ran_out) +
                                        " tiles, which were skipped; copies not seen to land: " +
                                        std::to_string(in_flight));
    return RR_OK;
}

rr_status_t rr_reducer_finish(rr_reducer_t* red, cudaStream_t stream)
{
    if (!red) return fail(RR_ERR_INVALID_ARG, "NULL reducer");
    for (size_t b = 0; b < red->pending.size(); ++b)
        if (red->pending[b] > 0) return fail(RR_ERR_INVALID_ARG, "a bucket still waits for gradients");
    cudaError_t e = cudaEventRecord(red->done, red->comm);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, red->done, 0);
    if (e != cudaSuccess) return cuda_fail(e, "joining the communication stream");
    red->reset();
    return RR_OK;
}

void rr_reducer_free(rr_reducer_t* red) { delete red; }

// ------------------------------------------------------ model, picker --

rr_status_t rr_cost_model(rr_algo_t algo, int nranks, double bytes, double alpha_s, double beta,
                          rr_cost_t* out)
{
    if (!out || nranks < 1 || beta <= 0) return fail(RR_ERR_INVALID_ARG, "bad cost-model arguments");
    const double n = nranks;
    rr_cost_t c{};
    switch (algo) {
    case RR_ALGO_RING:  // [P3] section 4: 2(N-1) steps, 2(N-1)/N M per rank
        c.steps = 2 * (n - 1);
        c.bytes_sent = 2 * (n - 1) / n * bytes;
        break;
    case RR_ALGO_TREE:  // [P3] section 6: 2 log2 N steps, the whole message per level
    {
        const double L = std::ceil(std::log2(n));
        c.steps = 2 * L;
        c.bytes_sent = 2 * L * bytes;
        break;
    }
    case RR_ALGO_ONESHOT:  // [P4]: one step, read every peer's buffer
    case RR_ALGO_TREE_ONESHOT:
        c.steps = nranks > 1 ? 1 : 0;
        c.bytes_sent = (n - 1) * bytes;
        break;
    case RR_ALGO_TWO_SHOT:  // [P4]: reduce-scatter then all-gather by direct reads
        c.steps = nranks > 1 ? 2 : 0;
        c.bytes_sent = 2 * (n - 1) / n * bytes;
        break;
    case RR_ALGO_DOUBLE_RING:  // [P3] section 6: half the bytes on each of two links
        c.steps = 2 * (n - 1);
        c.bytes_sent = (n - 1) / n * bytes;
        break;
    default:
        return fail(RR_ERR_INVALID_ARG, "unknown algo");
    }
    c.latency_s = c.steps * alpha_s;
    c.bandwidth_s = c.bytes_sent / beta;
    c.total_s = c.latency_s + c.bandwidth_s;
    *out = c;
    return RR_OK;
}

rr_status_t rr_set_picker_params(double launch_s, double hbm_bytes_per_s)
{
    if (launch_s == 0 && hbm_bytes_per_s == 0) {  // back to the measured table and the sweep's fit
        g_launch_s.store(kPickerAlphaS);
        g_hbm_bps.store(kPickerBetaBps);
        g_use_model.store(false);
        return RR_OK;
    }
    if (!(launch_s >= 0) || !(hbm_bytes_per_s > 0)) return fail(RR_ERR_INVALID_ARG, "bad picker parameters");
    g_launch_s.store(launch_s);
    g_hbm_bps.store(hbm_bytes_per_s);
    g_use_model.store(true);
    return RR_OK;
}

rr_algo_t rr_pick_algo(int nranks, size_t count, rr_dtype_t dtype)
{
    if (nranks <= 1) return RR_ALGO_ONESHOT;
    rr_algo_t a = RR_ALGO_AUTO;
    if (!g_use_model.load(std::memory_order_relaxed)) a = table_pick(nranks, (uint64_t)count * esize(dtype), 0);
    if (a == RR_ALGO_AUTO) a = model_pick(nranks, count, dtype);
    if (a == RR_ALGO_RING && (dtype == RR_BF16 || dtype == RR_F16)) a = RR_ALGO_ONESHOT;
    return a;
}

}  // extern "C"
