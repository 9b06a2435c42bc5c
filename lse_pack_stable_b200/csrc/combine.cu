// Stable log-sum-exp combine of a received packet (the step after the DCP
// all-to-all): recv_o [W_dst][W_src][N][D], recv_lse [W_dst][W_src][N].
#include "rowcombine.cuh"

namespace cplse {

cudaError_t launch_combine(const CombineArgs& a, Dtype dt, cudaStream_t s)
{
    return dt == Dtype::kBf16 ? launch_rowcombine_p<Bf16, kModeCombine>(a, s)
                              : launch_rowcombine_p<Fp16, kModeCombine>(a, s);
}

}  // namespace cplse
