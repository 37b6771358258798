// flex_fwd_d128_persist.cu -- persistent forward kernels for head dim 128 (no mask, sliding window).
#define FLEX_FWD_PERSISTENT_UNIT
#include "flex_fwd_inst.cuh"

namespace flexattn {
FLEX_FWD_PERSISTENT_INSTANCES(128)
}  // namespace flexattn
