/*
 * rr.h -- C ABI of the ring all-reduce library for N virtual ranks on one
 * NVIDIA B200 (sm_100a).
 *
 * A "virtual rank" is one device buffer in the GPU's HBM.  The library runs
 * the collectives that data-parallel training uses for gradient sync between
 * N such buffers: the ring all-reduce (a reduce-scatter of N chunks over N-1
 * ring steps, then an all-gather over N-1 steps), a fused one-shot all-reduce
 * that gives the ring's bits in one pass, tree-order variants, standalone
 * reduce-scatter, all-gather and all-to-all, and DDP-style gradient buckets.
 *
 * Sources (four web pages on ring all-reduce), cited by tag:
 *   [P1] "How all-reduce keeps every card identical" (mhpq.cn, news 451051)
 *   [P2] "AllReduce from principle to tuning" (xxqk.cn, news 376101)
 *   [P3] "Training gradient sync and collective communication: from parameter
 *        server to Ring AllReduce" (geek-doc.cn)
 *   [P4] "Collective communication primitives" (ai-infra-handbooks,
 *        train/basics/collectives)
 *
 * Conventions for every call below
 *   - Pointers named bufs/send/recv/grads/buckets are HOST arrays of DEVICE
 *     pointers, one per rank (nranks entries; grads has nranks*ntensors).
 *     The library copies the pointer values into kernel parameters and does
 *     not keep them.  The caller owns all device memory and the stream.
 *   - No call allocates device memory or synchronises the host; work is
 *     enqueued on `stream` and the call returns.  A CUDA launch error is
 *     returned as RR_ERR_CUDA (detail in rr_last_error()).
 *   - Argument errors are returned before anything is enqueued:
 *     RR_ERR_INVALID_ARG for a NULL, repeated or misaligned device pointer, nranks
 *     outside 1..RR_MAX_RANKS, overlapping buffers, a bad enum, an element
 *     count above 2^48 (far past any device memory; it keeps byte ranges
 *     from wrapping) or a count that the operation cannot split;
 *     RR_ERR_UNSUPPORTED for a valid but unsupported combination (AVG on
 *     int32).
 *   - count == 0 is RR_OK and enqueues nothing.  A device pointer must sit on
 *     a boundary of its element size (RR_ERR_INVALID_ARG otherwise); any such
 *     alignment is accepted.  Buffers whose addresses agree modulo 16 bytes
 *     take 128-bit vector or bulk-copy access after a scalar head per
 *     segment; a copy or conversion whose output sits at another 16-byte
 *     phase than its input is realigned through shared memory or across
 *     lanes; a one-shot or reduce-scatter over ranks at different phases
 *     stages every rank's tile at its own shift (the tree-order one-shot up
 *     to 16 ranks), and only the schedules' steps over ranks at different
 *     phases (one launch per step) and a tree-order one-shot over more ranks
 *     run element by element.
 *   - Chunking: chunk size C = ceil(count / N); chunk k is the element range
 *     [k*C, min((k+1)*C, count)), possibly short or empty ([P4] "Ring
 *     all-reduce and communication volume": the tensor is split with
 *     tensor.chunk(n)).
 *   - Reduction order ("ring order"): element i of chunk c = i / C reduces as
 *     ((x_c[i] op x_{c+1}[i]) op x_{c+2}[i]) ... op x_{c+N-1}[i], rank indices
 *     mod N, the partial on the left; this is the order in which the ring
 *     schedule folds chunk c (its partial starts on rank c and gains one rank
 *     per hop).  AVG is that SUM divided once by N.  MAX keeps the left
 *     operand unless it is smaller, MIN unless it is larger.
 *   - Precision: fp32, bf16 and fp16 reduce in fp32 ([P1] s5.3: reduce
 *     low-precision gradients in fp32); bf16 and fp16 results are rounded
 *     once to nearest-even, except in the RING, TREE and DOUBLE_RING
 *     schedules, whose partials live in the 16-bit buffers between steps and
 *     are rounded at every hop.  int32 SUM and PROD wrap modulo 2^32.
 */
#ifndef RR_H_
#define RR_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RR_MAX_RANKS 64
#define RR_VERSION 1

typedef enum rr_status {
    RR_OK = 0,
    RR_ERR_INVALID_ARG = 1,
    RR_ERR_UNSUPPORTED = 2,
    RR_ERR_CUDA = 3,
    RR_ERR_TIMEOUT = 4 /* a bounded device wait ran out (rr_check_timeouts) */
} rr_status_t;

/* Element types of the rank buffers: IEEE binary32, bfloat16 (the upper half
 * of a binary32), int32, IEEE binary16. */
typedef enum rr_dtype { RR_F32 = 0, RR_BF16 = 1, RR_I32 = 2, RR_F16 = 3 } rr_dtype_t;

/* Reductions of [P1] s2.1: SUM, AVG (sum then divide by N), MAX, MIN, PROD. */
typedef enum rr_op { RR_SUM = 0, RR_AVG = 1, RR_MAX = 2, RR_MIN = 3, RR_PROD = 4 } rr_op_t;

/* Algorithms.
 *   RING         the ring schedule ([P4] "Ring all-reduce and communication
 *                volume"; [P3] s3): its 2(N-1) steps in one launch when every
 *                buffer has the same 16-byte phase -- each CTA carries one
 *                tile of one chunk through all the steps in order, every step
 *                reading the neighbour's copy and writing its own as the
 *                schedule does (the same values, the same bytes) -- else one
 *                launch per step
 *   ONESHOT      one launch that reads all N buffers once, folds in ring
 *                order and writes the result to all N ([P4] "alpha-beta
 *                model": one-shot reads every peer's buffer directly)
 *   TREE         the tree schedule: ceil(log2 N) pairwise reduce levels,
 *                then as many broadcast levels ([P3] s6); one launch like
 *                RING (each CTA takes one tile through every level), else one
 *                launch per level
 *   TREE_ONESHOT one launch that folds in the tree's pairwise order
 *   TWO_SHOT     two launches: a reduce-scatter by direct reads (chunk c
 *                folded in ring order into its owner, rank c), then an
 *                all-gather by direct reads ([P4] "alpha-beta model": the
 *                two-shot all-reduce); the ring's bits and its 2(N-1)/N S
 *                bytes per rank, in 2 steps instead of 2(N-1)
 *   DOUBLE_RING  two rings in opposite directions at once ([P3] s6: the
 *                double ring): the first half of every buffer (H =
 *                ceil(count/2) elements) runs the RING schedule, the second
 *                half the mirror-image ring whose ranks send to the left, so
 *                a second-half chunk c folds downwards (c, c-1, ...); one
 *                launch like RING, else 2(N-1); each rank sends half its
 *                bytes each way
 *   AUTO         the picker's choice among RING, ONESHOT and TWO_SHOT
 *                (never a tree order or the double ring, whose bits differ);
 *                env RR_ALGO=ring|oneshot|tree|tree_oneshot|two_shot|
 *                double_ring overrides it. */
typedef enum rr_algo {
    RR_ALGO_AUTO = 0,
    RR_ALGO_RING = 1,
    RR_ALGO_ONESHOT = 2,
    RR_ALGO_TREE = 3,
    RR_ALGO_TREE_ONESHOT = 4,
    RR_ALGO_TWO_SHOT = 5,
    RR_ALGO_DOUBLE_RING = 6
} rr_algo_t;

/* The two phases of the ring ([P3] s3; [P4]). */
typedef enum rr_phase { RR_PHASE_REDUCE_SCATTER = 0, RR_PHASE_ALL_GATHER = 1 } rr_phase_t;

/* What the last call on this host thread did. */
typedef struct rr_stats {
    int32_t algo;              /* rr_algo_t that ran (never AUTO) */
    int32_t steps;             /* communication steps: ring 2(N-1), tree 2 ceil(log2 N), one-shot 1 */
    int32_t launches;          /* kernel launches enqueued */
    int32_t nranks;
    uint64_t bytes_per_rank;   /* S = count * element size */
    uint64_t bytes_sent_max;   /* most bytes any one rank sent (ring: 2(N-1)/N*S when N | count) */
    uint64_t bytes_sent_total; /* bytes sent by all ranks together */
    uint64_t hbm_bytes;        /* algorithmic HBM bytes read + written by the kernels */
    uint64_t host_ns;          /* host time of the call, entry to return (the library's share of the
                                  per-call cost the alpha-beta model calls alpha) */
    uint64_t launch_ns;        /* of which, time inside the kernel launch calls */
} rr_stats_t;

/* One transfer of the ring schedule: at (phase, step), `rank` sends chunk
 * send_idx to its right neighbour dst and receives chunk recv_idx from its
 * left neighbour; `bytes` is the size of the sent chunk. */
typedef struct rr_ring_event {
    int32_t phase;
    int32_t step;
    int32_t rank;
    int32_t dst;
    int32_t send_idx;
    int32_t recv_idx;
    uint64_t bytes;
} rr_ring_event_t;

/* Terms of the alpha-beta cost model ([P3] s4: T = 2(N-1) alpha +
 * 2(N-1)/N M / beta for the ring; [P4] "alpha-beta model"). */
typedef struct rr_cost {
    double steps;       /* sequential steps, each paying alpha */
    double bytes_sent;  /* bytes on the busiest rank's link */
    double latency_s;   /* steps * alpha */
    double bandwidth_s; /* bytes_sent / beta */
    double total_s;     /* latency_s + bandwidth_s */
} rr_cost_t;

/* ---------------------------------------------------------------- calls -- */

/* All-reduce in place over bufs[0..nranks): afterwards every buffer holds the
 * reduction of all inputs, element by element ([P4] "The five primitives";
 * [P1] s2.1).  count elements per rank.  Bits: RING, ONESHOT, TWO_SHOT and
 * AUTO give the ring order for fp32 and int32; for bf16 and fp16, ONESHOT,
 * TWO_SHOT and AUTO round once and RING rounds per hop.  TREE and
 * TREE_ONESHOT give the tree order; DOUBLE_RING the ring order in the first
 * half and the downward order in the second (rounding per hop for bf16 and
 * fp16).  Buffers must not
 * overlap.  nranks == 1 enqueues nothing. */
rr_status_t rr_allreduce(void* const* bufs, int nranks, size_t count, rr_dtype_t dtype, rr_op_t op,
                         rr_algo_t algo, cudaStream_t stream);

/* All-reduce of fp32 buffers with a low-precision wire ([P1] s7.3: represent
 * gradients in low precision to cut the communication volume): every value
 * that crosses a link -- each partial a reduce-scatter step sends, and each
 * finished chunk the all-gather sends -- is rounded to `wire` (RR_BF16, round
 * to nearest even), while every rank folds in fp32.  Element i of chunk c
 * gives acc = x_c; acc = bf16(acc) op x_{c+j} for j = 1..N-1; result =
 * bf16(acc, divided by N for AVG), the same value on every rank.  op: SUM or
 * AVG.  algo: RING (the 2(N-1)-step schedule with bf16 transfers) or
 * ONESHOT / AUTO (one launch, the same bits).  Error against the exact
 * reduction: at most about N * 2^-8 * sum |x|.  On one GPU the buffers stay
 * fp32 in HBM, so the HBM traffic is that of the fp32 call; the bytes counted
 * as sent (rr_get_stats) are the bf16 ones.  nranks == 1 sends nothing and
 * leaves the buffer unchanged. */
rr_status_t rr_allreduce_wire(void* const* bufs, int nranks, size_t count, rr_op_t op, rr_dtype_t wire,
                              rr_algo_t algo, cudaStream_t stream);

/* All-reduce of HOST buffers through caller-provided device buffers: copies
 * host_bufs[r] -> dev_bufs[r], reduces dev_bufs as rr_allreduce does, and
 * copies the result back into every host_bufs[r]; dev_bufs hold the result
 * too.  For the one-shot algorithms (AUTO's choice) above 8 MiB per rank the
 * work is pipelined in 8 MiB slices: uploads run on an internal stream,
 * folds on `stream`, downloads on a second internal stream, so uploads and
 * downloads overlap; the internal streams wait for `stream` first and
 * `stream` waits for them at the end, so the call is ordered on `stream`
 * like any other.  Host buffers should be page-locked for the copies to be
 * asynchronous.  Same arguments, results and errors as rr_allreduce; the
 * device buffers must not overlap.  The host buffers hold the result once
 * `stream` has been synchronised.  The first call on a device creates the two
 * streams and four events it keeps until exit. */
rr_status_t rr_allreduce_host(void* const* host_bufs, void* const* dev_bufs, int nranks, size_t count,
                              rr_dtype_t dtype, rr_op_t op, rr_algo_t algo, cudaStream_t stream);

/* The host-buffer all-reduce for callers that cannot allocate device memory.
 * The pages have no counterpart to this call: it exists for callers that
 * hold only host arrays and a stream and may not call cudaMalloc -- code that
 * runs while a framework's caching allocator holds all of the device's memory,
 * a plug-in that is handed no device buffers, or a latency-critical path that
 * must not call cudaMalloc or cudaFree because they can synchronise the device.
 * It does what rr_allreduce_host does with a caller's device buffers (copy
 * host_bufs[r] in, reduce, copy the result back into every host_bufs[r]; the
 * same bits), but stages the values in a region of device memory that the
 * library declares statically: RR_NOALLOC_MAX_BYTES (16 MiB) on every GPU that
 * loads the library, held until the process exits.  The call allocates
 * nothing, on the device or the host.
 *   - Limit: nranks slots of count elements, each rounded up to 256 bytes,
 *     must fit in RR_NOALLOC_MAX_BYTES; a larger call returns
 *     RR_ERR_INVALID_ARG before anything is enqueued.
 *   - algo: AUTO or ONESHOT (the one-shot all-reduce in ring order); others
 *     return RR_ERR_UNSUPPORTED.  Other arguments and errors as
 *     rr_allreduce_host; host buffers must not overlap.
 *   - The first call on a device looks up the staging region's device address
 *     there (cudaGetSymbolAddress, with that device current) and keeps it;
 *     make that first call before any stream capture on the device.
 *   - Every call on a device uses the same region, which keeps the last
 *     call's values; nothing in it needs to start at zero, because each call
 *     overwrites the bytes it reads.  Calls whose work overlaps on the GPU --
 *     on different streams, or from different threads, without ordering
 *     between them -- race on the region and give wrong results.
 *   - Host buffers should be page-locked for the copies to be asynchronous;
 *     they hold the result once `stream` has been synchronised. */
#define RR_NOALLOC_MAX_BYTES (16u << 20)
rr_status_t rr_allreduce_host_noalloc(void* const* host_bufs, int nranks, size_t count, rr_dtype_t dtype,
                                      rr_op_t op, rr_algo_t algo, cudaStream_t stream);

/* One step of the ring schedule for all ranks at once (one launch), in place:
 * reduce-scatter step s has every rank r fold chunk (r-s-1) mod N received
 * from rank r-1 into its own copy (received partial on the left; AVG divides
 * by N in step N-2); all-gather step s has every rank r overwrite chunk
 * (r-s) mod N with rank r-1's copy ([P4] ring_allreduce.py; [P3] s3, the
 * 4-GPU walkthrough).  step in 0..N-2.  Running the 2(N-1) steps in order is
 * exactly rr_allreduce(..., RR_ALGO_RING). */
rr_status_t rr_ring_step(void* const* bufs, int nranks, size_t count, rr_dtype_t dtype, rr_op_t op,
                         rr_phase_t phase, int step, cudaStream_t stream);

/* The ring schedule as data (host only): fills events[0..2(N-1)N) in the order
 * phase, step, rank -- exactly the transfers rr_ring_step launches.  *nevents
 * receives the number of events (also when capacity is too small, which
 * returns RR_ERR_INVALID_ARG). */
rr_status_t rr_ring_schedule(int nranks, size_t count, rr_dtype_t dtype, rr_ring_event_t* events,
                             size_t capacity, size_t* nevents);

/* Reduce-scatter ([P4] "The five primitives"; [P3] s6): send[p] holds
 * nranks*recvcount elements; recv[r] receives chunk r reduced over all ranks
 * in ring order (the fold of chunk r starts on rank r), so reduce-scatter
 * followed by all-gather equals the all-reduce bit for bit.  algo: AUTO or
 * ONESHOT (one launch).  recv buffers must not overlap the send buffers. */
rr_status_t rr_reduce_scatter(const void* const* send, void* const* recv, int nranks, size_t recvcount,
                              rr_dtype_t dtype, rr_op_t op, rr_algo_t algo, cudaStream_t stream);

/* All-gather ([P4] "The five primitives"): recv[r][p*sendcount + i] =
 * send[p][i] for every r and p.  algo: AUTO or ONESHOT (one launch: each
 * input element read once, written N times). */
rr_status_t rr_all_gather(const void* const* send, void* const* recv, int nranks, size_t sendcount,
                          rr_dtype_t dtype, rr_algo_t algo, cudaStream_t stream);

/* All-to-all ([P4] "The five primitives": rank r's p-th block goes to rank
 * p, a transpose): recv[r][p*C + i] = send[p][r*C + i], C = count_per_peer;
 * each buffer holds nranks*C elements.  Out of place, one launch. */
rr_status_t rr_all_to_all(const void* const* send, void* const* recv, int nranks, size_t count_per_peer,
                          rr_dtype_t dtype, cudaStream_t stream);

/* --------------------------------------------------------------- buckets -- */

/* Opaque bucket plan (host memory owned by the library). */
typedef struct rr_bucket_plan rr_bucket_plan_t;

/* DDP-style bucket plan ([P2] s3.3: gradients go into buckets in the order
 * given, and a bucket is reduced once it reaches the threshold; [P1] s5.2:
 * bucket_cap_mb, default 25).  Greedy over numels[0..ntensors) in the order
 * given, never splitting a tensor: each tensor joins the open bucket, which
 * closes as soon as its bytes (in grad_dtype) reach cap_bytes.  grad_dtype is
 * RR_BF16, RR_F16 or RR_F32; buckets are fp32.  Host only; free with
 * rr_bucket_plan_free. */
rr_status_t rr_bucket_plan(const size_t* numels, int ntensors, rr_dtype_t grad_dtype, size_t cap_bytes,
                           rr_bucket_plan_t** out);
void rr_bucket_plan_free(rr_bucket_plan_t* plan);

/* Plan queries (host only).  rr_bucket_info gives a bucket's first tensor,
 * its number of tensors and its length in fp32 elements; rr_bucket_tensor
 * gives a tensor's bucket and its element offset inside it. */
int rr_bucket_count(const rr_bucket_plan_t* plan);
rr_status_t rr_bucket_info(const rr_bucket_plan_t* plan, int bucket, int* first_tensor, int* ntensors,
                           size_t* numel);
rr_status_t rr_bucket_tensor(const rr_bucket_plan_t* plan, int tensor, int* bucket, size_t* offset);

/* Pack one bucket for every rank: buckets[r][offset(t) + j] = fp32(grads[r *
 * ntensors + t][j]) for each tensor t of the bucket (exact widening).  grads
 * holds nranks*ntensors device pointers (entries of tensors outside the
 * bucket are ignored); buckets holds nranks fp32 buffers of at least the
 * bucket's numel.  One launch. */
rr_status_t rr_bucket_pack(const rr_bucket_plan_t* plan, int bucket, const void* const* grads,
                           void* const* buckets, int nranks, cudaStream_t stream);

/* Unpack one reduced bucket: grads[r * ntensors + t][j] =
 * round(buckets[r][offset(t) + j] / N) for AVG (no division for SUM), one
 * round-to-nearest-even to the gradient dtype.  One launch. */
rr_status_t rr_bucket_unpack(const rr_bucket_plan_t* plan, int bucket, const void* const* buckets,
                             void* const* grads, int nranks, rr_op_t op, cudaStream_t stream);

/* Fused bucket sync: reduces one bucket's gradients across ranks in place,
 * with the bits of pack -> rr_allreduce(SUM, ring order over the bucket's
 * flat index) -> unpack(op), but reading and writing each gradient once
 * (4 bytes per bf16 parameter per rank instead of 20).  op: SUM or AVG.
 * One launch.  Where every rank's copy of a tensor shares a 16-byte phase
 * the launch is a programmatic dependent of the stream's previous kernel:
 * it waits for that kernel and its memory before reading, and a previous
 * sync of this library lets its CTAs be scheduled while it drains (so
 * back-to-back syncs of many buckets lose less to ramp-up); for syncs that
 * should run beside other work on the GPU, the reducer below launches
 * plainly. */
rr_status_t rr_bucket_allreduce(const rr_bucket_plan_t* plan, int bucket, void* const* grads,
                                int nranks, rr_op_t op, cudaStream_t stream);

/* Fused sync of buckets first_bucket .. first_bucket + nbuckets - 1 (a
 * gradient sync when every bucket is ready at once, e.g. without overlap):
 * the same bits as rr_bucket_allreduce on each bucket in turn -- every bucket
 * is still chunked over its own flat index -- but the buckets share launches
 * until a kernel parameter block is full (up to 384 tensors, 2048 gradient
 * pointers and 448 segments per launch), so the range costs a few launches
 * instead of one per bucket.  Same arguments and errors as
 * rr_bucket_allreduce; the range must lie inside the plan (RR_ERR_INVALID_ARG
 * otherwise) and every gradient it covers must be disjoint from the others.
 * Statistics cover the whole range. */
rr_status_t rr_bucket_allreduce_range(const rr_bucket_plan_t* plan, int first_bucket, int nbuckets,
                                      void* const* grads, int nranks, rr_op_t op, cudaStream_t stream);

/* ------------------------------------------------ overlapped bucket sync -- */

/* Opaque reducer (host memory and CUDA events owned by the library). */
typedef struct rr_reducer rr_reducer_t;

/* A DDP-style reducer: buckets are synced while backward still runs
 * ([P3] s5: backward produces gradients from the last layer to the first and
 * each bucket's all-reduce starts as soon as the bucket is ready, so the
 * communication hides behind the remaining backward; [P2] s3.3: each full
 * bucket triggers its all-reduce; [P1] s4.2).  Binds a plan (which must
 * outlive the reducer) to the gradients of all ranks -- grads holds
 * nranks*ntensors device pointers, rank-major, copied -- and to a
 * communication stream `comm`.  op: SUM or AVG.  max_ctas > 0 caps the CTAs
 * of each bucket sync (they then loop over the bucket's tiles), leaving the
 * other SMs to the kernels that produce the gradients, as a communication
 * library runs its collectives on a few channels; 0 launches one CTA per tile.
 * The gradients are checked here, once (RR_ERR_INVALID_ARG for a NULL or
 * overlapping one), so a step's syncs meet no argument error.
 * Creates one CUDA event per bucket plus one; allocates no device memory. */
rr_status_t rr_reducer_create(const rr_bucket_plan_t* plan, void* const* grads, int nranks, rr_op_t op,
                              cudaStream_t comm, int max_ctas, rr_reducer_t** out);

/* Marks tensor `tensor` (on every rank) as final once the work already
 * enqueued on `producer` has run.  When this completes its bucket, an event
 * is recorded on `producer`, `comm` waits for it and the bucket's fused sync
 * (rr_bucket_allreduce) is enqueued on `comm`.  The bucket's other tensors
 * must have been produced on `producer` too, or be ordered before it by the
 * caller.  RR_ERR_INVALID_ARG if the tensor was already marked in this
 * step. */
rr_status_t rr_reducer_ready(rr_reducer_t* red, int tensor, cudaStream_t producer);

/* Ends a step: `stream` waits for every bucket sync of the step, and the
 * marks are cleared for the next step.  RR_ERR_INVALID_ARG (and nothing
 * enqueued) if some tensor was not marked, i.e. its bucket was never
 * synced -- the situation in which DDP would hang. */
rr_status_t rr_reducer_finish(rr_reducer_t* red, cudaStream_t stream);
void rr_reducer_free(rr_reducer_t* red);

/* ----------------------------------------------------- picker and model -- */

/* The alpha-beta model of one algorithm for N ranks and M bytes per rank
 * ([P3] s4-s6; [P4] "alpha-beta model"): RING 2(N-1) steps moving 2(N-1)/N M
 * per rank; DOUBLE_RING 2(N-1) steps moving (N-1)/N M on each of a rank's two
 * links; TREE 2 ceil(log2 N) steps each moving M; ONESHOT 1 step in which
 * each rank reads (N-1) M; TWO_SHOT 2 steps moving 2(N-1)/N M.  alpha in seconds, beta in bytes/second. */
rr_status_t rr_cost_model(rr_algo_t algo, int nranks, double bytes_per_rank, double alpha_s,
                          double beta_bytes_per_s, rr_cost_t* out);

/* The algorithm AUTO runs for this call shape on 16-byte aligned buffers
 * (RING, ONESHOT or TWO_SHOT: the schedules whose results carry the ring's
 * bits).  It is measured, not modelled: a sweep of every candidate on the GPU
 * the library is built for gives a table of the fastest per (rank count, bytes
 * per rank, alignment class), and a call takes the nearest measured rank
 * count (in log2 ratio) and size ([P3] s4 and [P4] "alpha-beta model" say
 * which should win for small and large messages; the table is that
 * measurement).  AUTO itself also keys the table on the call's buffers:
 * 16-byte aligned, all at one other 16-byte phase, or at phases that differ.
 * bf16 and fp16 never take RING (its partials round at every hop).
 * rr_set_picker_params(alpha, beta) makes AUTO use the model instead -- the
 * rr_cost_model of one GPU, a launch costing alpha seconds and HBM moving beta
 * bytes per second -- and rr_set_picker_params(0, 0) returns to the table
 * (whose sweep also fitted the model's default alpha and beta). */
rr_algo_t rr_pick_algo(int nranks, size_t count, rr_dtype_t dtype);
rr_status_t rr_set_picker_params(double launch_s, double hbm_bytes_per_s);

/* ------------------------------------------------------------ utilities -- */

rr_status_t rr_get_stats(rr_stats_t* out); /* last call on this host thread */

/* Bounded waits.  The one-shot all-reduce (2-64 ranks), the reduce-scatter
 * (2-16 ranks), the tree-order one-shot (2-8, 12 and 16 ranks) and the fused
 * bucket sync (2-64 ranks) stage their tiles in shared memory with bulk async
 * copies when every rank's buffer sits at one 16-byte phase (on element
 * boundaries); their threads wait on an mbarrier for those
 * copies with an iteration limit instead of forever.  A wait that runs out --
 * no working device lets it -- makes the whole CTA skip its tile (nothing of
 * that tile's result is written) and is counted on the device; one thread
 * then waits once more, bounded, for the tile's copies to land, and counts
 * the tile a second time if they were not seen to land.  This call
 * synchronises the current device, takes both counts (atomically exchanged
 * for zero on the device) and returns RR_ERR_TIMEOUT if either is not zero
 * (rr_last_error() gives both), RR_OK otherwise.  No other kernel of the
 * library waits on anything. */
rr_status_t rr_check_timeouts(void);
const char* rr_status_string(rr_status_t status);
const char* rr_last_error(void); /* detail of the last failure on this thread */
int rr_version(void);

/* The compute capability the library's device code was built for, as the
 * CUDA runtime reports it for one of its kernels on the current device
 * (cudaFuncGetAttributes' binaryVersion: 100 for sm_100a), in *version.
 * RR_ERR_CUDA if the runtime cannot load the kernel there (no device, or one
 * the code was not built for). */
rr_status_t rr_binary_version(int* version);

#ifdef __cplusplus
}
#endif

#endif /* RR_H_ */
