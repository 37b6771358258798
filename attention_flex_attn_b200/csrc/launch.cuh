// launch.cuh -- host-side launchers shared between the translation units of the
// library: each forward (head dim, block mask) combination and the decode path is
// instantiated in a .cu file of its own so that they compile in parallel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "flex_attn.h"
#include "flex_bwd_sm100.cuh"
#include "flex_decode.cuh"
#include "flex_decode_gqa_tma.cuh"
#include "flex_fwd_fp8_sm100.cuh"
#include "flex_fwd_sm100.cuh"

namespace flexattn {

// Tensor maps of the 8-bit forward: Q [128, Sq, B*H], K [128, Skv, B*Hkv] and the
// transposed V^T [Skv_pad, 128, B*Hkv], all bytes, 128 x 128 boxes.
struct Fp8Maps {
  CUtensorMap q, k, vt;
};

// V transpose into vt, then the 8-bit forward over (score_mod, mask_mod, block mask)
// (flex_fwd_fp8.cu).
flex_status_t fp8_dispatch(int score, int mask, bool blocks, const uint8_t* v, uint8_t* vt, int64_t kv_rows,
                           const Fp8Maps& m, const Fp8Params& p, int n_units, cudaStream_t s);

// Forward over every (dtype, score_mod, mask_mod) instantiation of one head dim and
// block-mask mode.  Instantiated in flex_fwd_d{64,128}{,_blocks}.cu.
template <int D, bool BLOCKS>
flex_status_t fwd_dispatch(flex_dtype_t dtype, int score, int mask, const CUtensorMap& mq, const CUtensorMap& mk,
                           const CUtensorMap& mv, const FwdParams& p, int n_units, cudaStream_t s);

extern template flex_status_t fwd_dispatch<64, false>(flex_dtype_t, int, int, const CUtensorMap&,
                                                      const CUtensorMap&, const CUtensorMap&, const FwdParams&,
                                                      int, cudaStream_t);
extern template flex_status_t fwd_dispatch<128, false>(flex_dtype_t, int, int, const CUtensorMap&,
                                                       const CUtensorMap&, const CUtensorMap&, const FwdParams&,
                                                       int, cudaStream_t);
extern template flex_status_t fwd_dispatch<64, true>(flex_dtype_t, int, int, const CUtensorMap&,
                                                     const CUtensorMap&, const CUtensorMap&, const FwdParams&,
                                                     int, cudaStream_t);
extern template flex_status_t fwd_dispatch<128, true>(flex_dtype_t, int, int, const CUtensorMap&,
                                                      const CUtensorMap&, const CUtensorMap&, const FwdParams&,
                                                      int, cudaStream_t);

// Tensor maps of the backward: Q and dO [D, Sq, B*H], K and V [D, Skv, B*Hkv].
struct BwdMaps {
  CUtensorMap q, o, k, v;
};

// Backward (prep, dQ, dK/dV; with a block mask also the transposed bitmaps) over every
// (dtype, score_mod, mask_mod) of one head dim and block-mask mode.  Instantiated in
// flex_bwd_d{64,128}{,_blocks}.cu.
template <int D, bool BLOCKS>
flex_status_t bwd_dispatch(flex_dtype_t dtype, int score, int mask, const BwdMaps& m, const BwdParams& p,
                           cudaStream_t s);
extern template flex_status_t bwd_dispatch<64, false>(flex_dtype_t, int, int, const BwdMaps&, const BwdParams&,
                                                      cudaStream_t);
extern template flex_status_t bwd_dispatch<128, false>(flex_dtype_t, int, int, const BwdMaps&, const BwdParams&,
                                                       cudaStream_t);
extern template flex_status_t bwd_dispatch<64, true>(flex_dtype_t, int, int, const BwdMaps&, const BwdParams&,
                                                     cudaStream_t);
extern template flex_status_t bwd_dispatch<128, true>(flex_dtype_t, int, int, const BwdMaps&, const BwdParams&,
                                                      cudaStream_t);

// Tensor maps of the caches ([D, cap, B*Hkv], 64 x 64 boxes) and of the additive mask
// ([cap, H, B], 64 x mask_rows boxes; mask_rows = 0: the mask is read directly), and the
// persistent grid of the grouped-query decode.
struct DecodeMaps {
  CUtensorMap k, v, m;
  int mask_rows;
  int grid;
};

// Split-KV decode + combine (flex_decode_launch.cu).  maps: the grouped-query decode's
// tensor maps (G >= 2), or nullptr for the register-streaming kernels.
flex_status_t decode_dispatch(int D, flex_dtype_t dtype, const DecodeParams& p, const DecodeMaps* maps,
                              cudaStream_t s);

}  // namespace flexattn
