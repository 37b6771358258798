// flex_bwd_d128.cu -- backward kernels (prep, dQ, dK/dV) for head dim 128.
#include "flex_bwd_inst.cuh"

namespace flexattn {
template flex_status_t bwd_dispatch<128, false>(flex_dtype_t, int, int, const BwdMaps&, const BwdParams&,
                                               cudaStream_t);
}  // namespace flexattn
