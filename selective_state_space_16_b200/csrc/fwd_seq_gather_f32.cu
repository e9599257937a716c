// fwd_seq_gather_f32.cu -- instantiation of the sequential forward family that gathers rows
// whose byte length is not a multiple of 16 itself, for f32 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_gather<float>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
