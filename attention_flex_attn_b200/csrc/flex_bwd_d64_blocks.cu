// flex_bwd_d64_blocks.cu -- backward kernels for head dim 64 with a block mask (the
// transpose pre-pass, prep, dQ, dK/dV).
#include "flex_bwd_inst.cuh"

namespace flexattn {
template flex_status_t bwd_dispatch<64, true>(flex_dtype_t, int, int, const BwdMaps&, const BwdParams&,
                                              cudaStream_t);
}  // namespace flexattn
