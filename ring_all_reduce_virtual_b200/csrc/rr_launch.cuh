// rr_launch.cuh -- launch helpers shared by the kernel files: one CTA per
// work item, and the dispatch from (dtype, op) codes to kernel templates.
#pragma once

#include <type_traits>

#include "rr_device.cuh"
#include "rr_internal.h"

namespace rr {

// One CTA per work item, up to the grid limit.  (A grid of one wave of
// resident CTAs looping over the tiles measured about 15 % slower on the
// 8 x 256 MiB all-reduce.)
template <class P>
inline cudaError_t launch_all(void (*kernel)(P), const P& p, uint64_t work, cudaStream_t s)
{
    if (work == 0) return cudaSuccess;
    const uint64_t grid = work < kMaxGrid ? work : kMaxGrid;
    kernel<<<(unsigned)grid, kThreads, 0, s>>>(p);
    return cudaGetLastError();
}

template <class F>
inline cudaError_t with_type(int dtype, int op, F&& f)
{
    auto by_op = [&]<class Ty>() -> cudaError_t {
        switch (op) {
        case kSum: return f.template operator()<Ty, kSum>();
        case kMax: return f.template operator()<Ty, kMax>();
        case kMin: return f.template operator()<Ty, kMin>();
        case kProd: return f.template operator()<Ty, kProd>();
        case kAvg:
            if constexpr (std::is_same_v<Ty, I32T>) return cudaErrorInvalidValue;
            else return f.template operator()<Ty, kAvg>();
        }
        return cudaErrorInvalidValue;
    };
    switch (dtype) {
    case kF32: return by_op.template operator()<F32T>();
    case kBF16: return by_op.template operator()<BF16T>();
    case kF16: return by_op.template operator()<F16T>();
    case kI32: return by_op.template operator()<I32T>();
    }
    return cudaErrorInvalidValue;
}

}  // namespace rr
