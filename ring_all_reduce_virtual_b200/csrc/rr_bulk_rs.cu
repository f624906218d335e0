// rr_bulk_rs.cu -- the bulk-copy reduce-scatter: part r of every rank staged
// in shared memory by bulk async copies, folded in ring order from rank r
// (the all-reduce's order for chunk r, so reduce-scatter then all-gather
// equals the all-reduce bit for bit), written to out[r].  Kernel template in
// rr_bulk.cuh; eligibility in rr_bulk.cu.
//
// Sources: [P4] "Collective communication primitives" (ai-infra-handbooks),
// sections "The five primitives" and "Ring all-reduce and communication
// volume".
#include "rr_bulk.cuh"

namespace rr {

template <class Ty, int OP>
cudaError_t launch_scatter_bulk(const RankParams& p, cudaStream_t s)
{
    switch (p.n) {
    case 2: return launch_bulk_fold<Ty, OP, 2, kBulkScatter, 0>(p, p.C, s);
    case 4: return launch_bulk_fold<Ty, OP, 4, kBulkScatter, 0>(p, p.C, s);
    case 8: return launch_bulk_fold<Ty, OP, 8, kBulkScatter, 0>(p, p.C, s);
    case 16: return launch_bulk_fold<Ty, OP, 16, kBulkScatter, 0>(p, p.C, s);
    }
    return launch_bulk_fold<Ty, OP, 0, kBulkScatter, 0>(p, p.C, s);
}

#define RR_INSTANTIATE(TY, OP) template cudaError_t launch_scatter_bulk<TY, OP>(const RankParams&, cudaStream_t);
RR_FOR_EACH_TYPE_OP(RR_INSTANTIATE)
#undef RR_INSTANTIATE

}  // namespace rr
