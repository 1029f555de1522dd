// Backward row kernels for bf16 rows, every activation and team shape.  Each
// direction and element format is its own unit so that the library's units
// compile in parallel; the kernels themselves are in rn_rows.cuh.
#include "rn_rows.cuh"

namespace rn_detail {
template rn_status launch_bwd<RN_BF16>(int, bool, const Sched&, int, const BwdArgs&, int64_t,
                                        cudaStream_t);
}  // namespace rn_detail
