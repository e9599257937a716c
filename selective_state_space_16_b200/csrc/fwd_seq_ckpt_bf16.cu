// fwd_seq_ckpt_bf16.cu -- instantiation of the sequential forward family storing checkpoints
// for the backward, for bf16 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_ckpt<__nv_bfloat16>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
