// fwd_seq_flagged_f32.cu -- instantiation of the sequential forward family
// (zero-order hold and / or conv prologue) for f32 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_flagged<float>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
