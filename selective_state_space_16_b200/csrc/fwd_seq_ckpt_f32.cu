// fwd_seq_ckpt_f32.cu -- instantiation of the sequential forward family storing checkpoints
// for the backward, for f32 I/O.
#include "launch_seq.cuh"

namespace ssmh {
template ssm_status_t launch_seq_ckpt<float>(const FwdArgs&, const ssm_fwd_options_t&);
}  // namespace ssmh
