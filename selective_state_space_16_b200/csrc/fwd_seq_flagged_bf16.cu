// fwd_seq_flagged_bf16.cu -- instantiation of the sequential forward family
// (zero-order hold and / or conv prologue) for bf16 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_flagged<__nv_bfloat16>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
