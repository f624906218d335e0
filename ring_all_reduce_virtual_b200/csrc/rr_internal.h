// rr_internal.h -- kernel parameter blocks and launchers shared between the
// host dispatcher (rr_api.cu) and the kernels (rr_kernels.cu, rr_bucket.cu).
// Not part of the C ABI.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

namespace rr {

constexpr int kMaxRanksH = 64;

// Rule-driven collectives over N rank buffers (one-shot all-reduce in ring
// or tree order, reduce-scatter, all-gather, all-to-all).
struct RankParams {
    const void* in[kMaxRanksH];
    void* out[kMaxRanksH];
    int n;          // ranks
    int vec_ok;     // all in[] agree modulo 16 bytes, and all out[] do
    float divisor;  // AVG's divisor (the rank count)
    int pad_;
    uint64_t C;     // chunk / part length in elements
    uint64_t count; // elements per rank buffer (all-reduce)
    uint64_t nseg;  // segments
    uint64_t tps;   // tiles per segment
    uint64_t lo;    // one-shot all-reduce: element range [lo, hi) of every
    uint64_t hi;    //   rank processed by this launch
    int owner_only; // one-shot all-reduce: write chunk c only to rank c (two-shot's first shot)
    int pad2_;
    unsigned int* waits;  // the bulk-copy kernels' wait counters on the launching device
                          // (bulk_wait_counters(); NULL keeps a call off those kernels)
};

// One segment of a table-driven step (a ring step, a tree level): fold
// in0 op in1 (in0 on the left) into out, or copy in0 into out when the step
// has one input.
struct StepSeg {
    const void* in0;
    const void* in1;
    void* out;
    uint64_t len;
};

struct StepParams {
    StepSeg seg[2 * kMaxRanksH];  // one per rank, or two (the double ring's two directions)
    int nseg;
    int nin;        // 2: fold, 1: copy
    int vec_ok;     // every segment's pointers agree modulo 16 bytes
    float divisor;  // AVG's divisor when this step finishes the fold
    uint64_t tps;
};

// The ring, double-ring and tree schedules in one launch.  The schedules'
// data dependencies run along (chunk, tile) chains: tile t of chunk k at
// ring step s reads only what step s-1 wrote to tile t of chunk k (on the
// previous rank), and a tree level reads only what the level below wrote to
// the same elements.  So one CTA carries its tile through every step, each
// thread on the same elements at every step (it reads what it wrote itself),
// and no CTA waits for another.
struct ChainParams {
    void* buf[kMaxRanksH];
    int n;
    int vec_ok;      // every buffer at the same 16-byte phase (required: the chains run the vector path)
    float divisor;   // AVG's divisor
    int nhalf;       // ring: 1 (the whole buffer, clockwise); double ring: 2 (half 1 counter-clockwise)
    uint64_t count;  // elements per rank
    uint64_t H;      // the double ring's first element of half 1 (count for the ring)
    uint64_t C[2];   // chunk size of each half
    uint64_t tps;    // tiles per chunk (ring) or per buffer (tree)
};

// Bucket launches: one launch covers up to kMaxBucketTensors tensors of one
// bucket and up to kMaxBucketPtrs gradient pointers (tensor-major: entry
// t * n + r is rank r's copy of the launch's t-th tensor).
constexpr int kMaxBucketPtrs = 2048;
constexpr int kMaxBucketTensors = 384;
constexpr int kMaxBucketSegs = kMaxBucketTensors + kMaxRanksH;

// Work items of the bucket kernels are numbered through per-segment prefix
// sums of their tile counts, so segments of very different lengths launch no
// empty CTAs: work item w belongs to the segment s with
// tile0[s] <= w < tile0[s + 1].
struct BucketCopyParams {
    const void* grad[kMaxBucketPtrs];      // pack: sources; unpack: destinations
    void* bucket[kMaxRanksH];              // fp32 bucket of each rank
    uint64_t toff[kMaxBucketTensors];      // element offset of tensor t in the bucket
    uint64_t tlen[kMaxBucketTensors];      // elements of tensor t
    uint64_t tile0[kMaxBucketTensors + 1]; // first work item of tensor t (n ranks x its tiles)
    int n;
    int nt;
    float divisor;
    int pad_;
};

// A fused bucket segment: elements [off, off + len) of launch tensor t, all
// in the bucket's chunk c (their fold starts on rank c).
struct BucketSeg {
    uint32_t t;
    uint32_t c;
    uint64_t off;
    uint64_t len;
};

struct BucketFoldParams {
    void* grad[kMaxBucketPtrs];
    BucketSeg seg[kMaxBucketSegs];
    uint64_t tile0[kMaxBucketSegs + 1];  // first work item (tile) of segment s
    int n;
    int nseg;
    int vec_ok;
    float divisor;
};

enum DType : int { kF32 = 0, kBF16 = 1, kI32 = 2, kF16 = 3 };
enum Kind : int {
    kOneshotRing = 0,
    kOneshotTree = 1,
    kReduceScatter = 2,
    kAllGather = 3,
    kAllToAll = 4,
    kChunkBroadcast = 5  // chunk c of rank c copied to chunk c of every other rank
};

// Vectors per thread per tile: kernels that fold N inputs keep N loads per
// vector in flight and use few vectors; kernels with one or two inputs use
// more vectors to keep as many loads in flight.
constexpr int kVptReduce = 2;
constexpr int kVptMove = 4;

// Vectors per thread of the N-input folds (one-shot all-reduce, reduce-scatter,
// fused bucket sync, tree-order one-shot).  These kernels are also compiled for
// fixed rank counts (2, 3, 4, 8, 16; the bucket kernel 2, 4, 8): with the
// count known the compiler unrolls every rank loop, needs few registers and
// keeps N * 2 loads per thread in flight at high occupancy.  Other counts run
// a variant with a runtime rank count.
inline int reduce_vpt(int) { return kVptReduce; }

// Elements one fold tile covers (for sizing tiles per segment on the host),
// and one bucket pack/unpack tile.
uint64_t tile_elems(int dtype, int vpt);
uint64_t bucket_tile_elems(int grad_dtype);

// Launch configuration: one CTA per work item (a tile of a segment), up to
// the grid limit; kernels loop over the rest.
constexpr uint64_t kMaxGrid = 0x7fffffffull;

// Launchers: return the launch's cudaError_t.  `op` is an rr_op_t value.
cudaError_t launch_rank_kernel(int kind, int dtype, int op, const RankParams& p, cudaStream_t s);
cudaError_t launch_step(int dtype, int op, const StepParams& p, cudaStream_t s);
// The whole ring schedule (p.nhalf 1) or double ring (2) in one launch, and
// the whole tree schedule (reduce levels, then broadcast levels) in one launch;
// wire: the ring's bf16 wire format (fp32 buffers, SUM or AVG).
cudaError_t launch_ring_chain(int dtype, int op, bool wire, const ChainParams& p, cudaStream_t s);
uint64_t chain_tile_elems(int dtype);  // elements of one chain tile (ChainParams::tps counts these)
cudaError_t launch_tree_chain(int dtype, int op, const ChainParams& p, cudaStream_t s);
// bf16 wire (fp32 buffers, SUM or AVG): the fused one-shot, and a reduce-scatter
// step (wire 1: the step completes its chunks; 2: it does not).
cudaError_t launch_oneshot_wire(int op, const RankParams& p, uint64_t work, cudaStream_t s);
cudaError_t launch_step_wire(int op, int wire, const StepParams& p, cudaStream_t s);
// The bulk-copy kernels' two wait counters on the current device (tiles whose
// bounded wait ran out; of those, tiles whose copies were not seen to land),
// looked up once per device; NULL if the lookup fails.
unsigned int* bulk_wait_counters();
// Takes (reads and clears, atomically on the device) both counters of the
// current device.  Synchronous.
cudaError_t take_bulk_timeouts(unsigned int* ran_out, unsigned int* in_flight);
// cudaFuncGetAttributes(...).binaryVersion of one of the library's kernels.
cudaError_t kernel_binary_version(int* version);
cudaError_t launch_bucket_pack(int grad_dtype, const BucketCopyParams& p, cudaStream_t s);
cudaError_t launch_bucket_unpack(int grad_dtype, int op, const BucketCopyParams& p, cudaStream_t s);
// pdl: launch the bulk-copy sync as a programmatic dependent of the stream's
// previous kernel (its CTAs scheduled while a previous sync drains): for
// back-to-back syncs, not for syncs that run beside other work (the reducer),
// whose waiting CTAs would hold SMs that work could use.
cudaError_t launch_bucket_fold(int grad_dtype, int op, const BucketFoldParams& p, cudaStream_t s,
                               uint64_t max_grid = kMaxGrid, bool pdl = false);

}  // namespace rr

namespace rr {
// Kernel parameter blocks must fit the 32,764-byte kernel parameter limit.
static_assert(sizeof(RankParams) <= 32764, "RankParams too large");
static_assert(sizeof(StepParams) <= 32764, "StepParams too large");
static_assert(sizeof(ChainParams) <= 32764, "ChainParams too large");
static_assert(sizeof(BucketCopyParams) <= 32764, "BucketCopyParams too large");
static_assert(sizeof(BucketFoldParams) <= 32764, "BucketFoldParams too large");
}  // namespace rr
