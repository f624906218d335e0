// rr_bulk_tree.cu -- the bulk-copy one-shot in the tree's pairwise order:
// every rank's tile staged in shared memory by bulk async copies, folded
// pairwise with fp32 partials (the same order and bits as
// oneshot_tree_kernel), written to every rank; 2-8, 12 and 16 ranks.
// Kernel template in rr_bulk.cuh; eligibility in rr_bulk.cu.
//
// Sources: [P3] "Training gradient sync and collective communication"
// (geek-doc.cn), section 6 (tree reduction: ranks pair up, pairs pair up).
#include "rr_bulk.cuh"

namespace rr {

template <class Ty, int OP>
cudaError_t launch_tree_bulk(const RankParams& p, cudaStream_t s)
{
    switch (p.n) {
    case 2: return launch_bulk_fold<Ty, OP, 2, kBulkTree, 0>(p, p.count, s);
    case 3: return launch_bulk_fold<Ty, OP, 3, kBulkTree, 0>(p, p.count, s);
    case 4: return launch_bulk_fold<Ty, OP, 4, kBulkTree, 0>(p, p.count, s);
    case 5: return launch_bulk_fold<Ty, OP, 5, kBulkTree, 0>(p, p.count, s);
    case 6: return launch_bulk_fold<Ty, OP, 6, kBulkTree, 0>(p, p.count, s);
    case 7: return launch_bulk_fold<Ty, OP, 7, kBulkTree, 0>(p, p.count, s);
    case 8: return launch_bulk_fold<Ty, OP, 8, kBulkTree, 0>(p, p.count, s);
    case 12: return launch_bulk_fold<Ty, OP, 12, kBulkTree, 0>(p, p.count, s);
    case 16: return launch_bulk_fold<Ty, OP, 16, kBulkTree, 0>(p, p.count, s);
    }
    return cudaErrorInvalidValue;
}

#define RR_INSTANTIATE(TY, OP) template cudaError_t launch_tree_bulk<TY, OP>(const RankParams&, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_INSTANTIATE)
#undef RR_INSTANTIATE

}  // namespace rr
