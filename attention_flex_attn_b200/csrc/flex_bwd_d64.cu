// flex_bwd_d64.cu -- backward kernels (prep, dQ, dK/dV) for head dim 64.
#include "flex_bwd_inst.cuh"

namespace flexattn {
template flex_status_t bwd_dispatch<64, false>(flex_dtype_t, int, int, const BwdMaps&, const BwdParams&,
                                               cudaStream_t);
}  // namespace flexattn
