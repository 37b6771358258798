// flex_fwd_d64.cu -- forward kernels for head dim 64, key tiles from the ranges mask_mod implies.
#include "flex_fwd_inst.cuh"

namespace flexattn {
template flex_status_t fwd_dispatch<64, false>(flex_dtype_t, int, int, const CUtensorMap&, const CUtensorMap&,
                                              const CUtensorMap&, const FwdParams&, int, cudaStream_t);
}  // namespace flexattn
