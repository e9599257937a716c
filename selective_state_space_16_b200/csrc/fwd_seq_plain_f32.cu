// fwd_seq_plain_f32.cu -- instantiation of the sequential forward family
// (plain discretisation, no conv) for f32 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_plain<float>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
