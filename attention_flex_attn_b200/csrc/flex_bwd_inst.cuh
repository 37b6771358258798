// flex_bwd_inst.cuh -- body of the backward instantiation units: the backward launches
// for one head dim and block-mask mode, dispatched over (dtype, score_mod, mask_mod).
// Included by flex_bwd_d{64,128}{,_blocks}.cu.
#pragma once

#include <atomic>
#include <cstdint>

#include "flex_bwd_sm100.cuh"
#include "launch.cuh"

namespace flexattn {
namespace {

template <int D, typename T, int SCORE, int MASK, bool BLOCKS, int WHICH, typename K>
bool bwd_smem_attr(K kernel, int bytes) {
  static std::atomic<uint64_t> done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
  done.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

template <int D, typename T, int SCORE, int MASK, bool BLOCKS>
flex_status_t launch_bwd(const BwdMaps& m, const BwdParams& p, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.Sq_pad;
  const int prep_blocks = static_cast<int>((rows * 32 + 255) / 256 < 148 * 16 ? (rows * 32 + 255) / 256 : 148 * 16);
  bwd_prep_kernel<D, T><<<prep_blocks, 256, 0, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FLEX_ERR_CUDA;
  if constexpr (BLOCKS) {
    // the transposed block mask: zeroed, then one bit per listed (query tile, key tile)
    const size_t bytes = static_cast<size_t>(p.B) * p.Hkv * p.n_ktiles * 2 * p.tb_words * sizeof(uint32_t);
    if (cudaMemsetAsync(p.tbits, 0, bytes, s) != cudaSuccess) return FLEX_ERR_CUDA;
    const int64_t lrows = static_cast<int64_t>(p.B) * p.H * p.n_qtiles;
    const int tb_blocks = static_cast<int>((lrows * 32 + 255) / 256 < 148 * 16 ? (lrows * 32 + 255) / 256 : 148 * 16);
    bwd_block_transpose_kernel<MASK><<<tb_blocks, 256, 0, s>>>(p);
    if (cudaGetLastError() != cudaSuccess) return FLEX_ERR_CUDA;
  }
  auto kq = bwd_dq_kernel<D, T, SCORE, MASK, BLOCKS>;
  if (!bwd_smem_attr<D, T, SCORE, MASK, BLOCKS, 0>(kq, BwdDqSmem<D, BLOCKS>::kAlloc)) return FLEX_ERR_CUDA;
  kq<<<p.B * p.H * p.n_qtiles, kBwdThreads, BwdDqSmem<D, BLOCKS>::kAlloc, s>>>(m.q, m.o, m.k, m.v, p);
  if (cudaGetLastError() != cudaSuccess) return FLEX_ERR_CUDA;
  auto kkv = bwd_dkdv_kernel<D, T, SCORE, MASK, BLOCKS>;
  if (!bwd_smem_attr<D, T, SCORE, MASK, BLOCKS, 1>(kkv, BwdDkvSmem<D>::kAlloc)) return FLEX_ERR_CUDA;
  kkv<<<p.B * p.Hkv * p.n_ktiles, kBwdThreads, BwdDkvSmem<D>::kAlloc, s>>>(m.q, m.o, m.k, m.v, p);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

template <int D, typename T, int SCORE, bool BLOCKS>
flex_status_t bwd_mask(int mask, const BwdMaps& m, const BwdParams& p, cudaStream_t s) {
  switch (mask) {
    case kMaskNone: return launch_bwd<D, T, SCORE, kMaskNone, BLOCKS>(m, p, s);
    case kMaskCausal: return launch_bwd<D, T, SCORE, kMaskCausal, BLOCKS>(m, p, s);
    case kMaskSliding: return launch_bwd<D, T, SCORE, kMaskSliding, BLOCKS>(m, p, s);
    case kMaskOffset: return launch_bwd<D, T, SCORE, kMaskOffset, BLOCKS>(m, p, s);
    case kMaskDocument: return launch_bwd<D, T, SCORE, kMaskDocument, BLOCKS>(m, p, s);
    case kMaskDocumentCausal: return launch_bwd<D, T, SCORE, kMaskDocumentCausal, BLOCKS>(m, p, s);
  }
  return FLEX_ERR_INVALID_ARG;
}

template <int D, typename T, bool BLOCKS>
flex_status_t bwd_score(int score, int mask, const BwdMaps& m, const BwdParams& p, cudaStream_t s) {
  if (score == kScoreNone) return bwd_mask<D, T, kScoreNone, BLOCKS>(mask, m, p, s);
  return bwd_mask<D, T, kScoreAlibi, BLOCKS>(mask, m, p, s);
}

}  // namespace

template <int D, bool BLOCKS>
flex_status_t bwd_dispatch(flex_dtype_t dtype, int score, int mask, const BwdMaps& m, const BwdParams& p,
                           cudaStream_t s) {
  if (dtype == FLEX_DTYPE_BF16) return bwd_score<D, __nv_bfloat16, BLOCKS>(score, mask, m, p, s);
  return bwd_score<D, __half, BLOCKS>(score, mask, m, p, s);
}

}  // namespace flexattn
