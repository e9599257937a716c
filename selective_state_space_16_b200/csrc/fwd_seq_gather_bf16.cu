// fwd_seq_gather_bf16.cu -- instantiation of the sequential forward family that gathers rows
// whose byte length is not a multiple of 16 itself, for bf16 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_gather<__nv_bfloat16>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
