// Forward row kernels for fp16 rows, every activation and team shape.  Each
// direction and element format is its own unit so that the library's units
// compile in parallel; the kernels themselves are in rn_rows.cuh.
#include "rn_rows.cuh"

namespace rn_detail {
template rn_status launch_fwd<RN_F16>(int, bool, const Sched&, const FwdArgs&, cudaStream_t);
}  // namespace rn_detail
