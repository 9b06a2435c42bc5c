// Fused pack -> all-to-all -> stable combine: destination j's output row
// (t, hc) reads row (t, j*Hc + hc) of every rank's partial output and
// statistics in place, so the packet never exists in HBM. Same arithmetic,
// in the same order, as pack (LSE formation) followed by combine.
#include "rowcombine.cuh"

namespace cplse {

cudaError_t launch_fused(const CombineArgs& a, Dtype dt, cudaStream_t s)
{
    return dt == Dtype::kBf16 ? launch_rowcombine_p<Bf16, kModeFused>(a, s)
                              : launch_rowcombine_p<Fp16, kModeFused>(a, s);
}

}  // namespace cplse
