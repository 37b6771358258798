// flex_fwd_d128_blocks.cu -- forward kernels for head dim 128, key tiles from a block mask.
#include "flex_fwd_inst.cuh"

namespace flexattn {
template flex_status_t fwd_dispatch<128, true>(flex_dtype_t, int, int, const CUtensorMap&, const CUtensorMap&,
                                              const CUtensorMap&, const FwdParams&, int, cudaStream_t);
}  // namespace flexattn
