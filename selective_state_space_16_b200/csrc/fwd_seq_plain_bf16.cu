// fwd_seq_plain_bf16.cu -- instantiation of the sequential forward family
// (plain discretisation, no conv) for bf16 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_plain<__nv_bfloat16>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
