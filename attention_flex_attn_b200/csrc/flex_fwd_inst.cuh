// flex_fwd_inst.cuh -- body of the forward instantiation units: sets the shared-memory
// attribute once per kernel and device, and dispatches (dtype, score_mod, mask_mod)
// onto the compile-time specialised kernels.  Included by flex_fwd_d*.cu only, each of
// which instantiates fwd_dispatch for one (head dim, block mask) pair.
#pragma once

#include <atomic>
#include <cstdint>

#include "launch.cuh"

namespace flexattn {
namespace {

// Per-device "attribute already set" bits, one set per kernel instantiation (the tag
// parameters make every instantiation own its static).
template <int D, typename T, int SCORE, int MASK, bool BLOCKS, typename K>
bool ensure_smem_attr(K kernel, int bytes) {
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
flex_status_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdParams& p,
                         int n_units, cudaStream_t stream) {
  auto kern = flex_fwd_kernel<D, T, SCORE, MASK, BLOCKS>;
  constexpr int kSmem = FwdSmem<D, BLOCKS, is_doc_mask(MASK)>::kAlloc;
  if (!ensure_smem_attr<D, T, SCORE, MASK, BLOCKS>(kern, kSmem)) return FLEX_ERR_CUDA;
  kern<<<n_units, kFwdThreads, kSmem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

template <int D, typename T, int SCORE, bool BLOCKS>
flex_status_t dispatch_mask(int mask, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const FwdParams& p, int n_units, cudaStream_t s) {
  switch (mask) {
    case kMaskNone: return launch_fwd<D, T, SCORE, kMaskNone, BLOCKS>(mq, mk, mv, p, n_units, s);
    case kMaskCausal: return launch_fwd<D, T, SCORE, kMaskCausal, BLOCKS>(mq, mk, mv, p, n_units, s);
    case kMaskSliding: return launch_fwd<D, T, SCORE, kMaskSliding, BLOCKS>(mq, mk, mv, p, n_units, s);
    case kMaskOffset: return launch_fwd<D, T, SCORE, kMaskOffset, BLOCKS>(mq, mk, mv, p, n_units, s);
    case kMaskDocument: return launch_fwd<D, T, SCORE, kMaskDocument, BLOCKS>(mq, mk, mv, p, n_units, s);
    case kMaskDocumentCausal:
      return launch_fwd<D, T, SCORE, kMaskDocumentCausal, BLOCKS>(mq, mk, mv, p, n_units, s);
  }
  return FLEX_ERR_INVALID_ARG;
}

template <int D, typename T, bool BLOCKS>
flex_status_t dispatch_score(int score, int mask, const CUtensorMap& mq, const CUtensorMap& mk,
                             const CUtensorMap& mv, const FwdParams& p, int n_units, cudaStream_t s) {
  if (score == kScoreNone) return dispatch_mask<D, T, kScoreNone, BLOCKS>(mask, mq, mk, mv, p, n_units, s);
  return dispatch_mask<D, T, kScoreAlibi, BLOCKS>(mask, mq, mk, mv, p, n_units, s);
}

}  // namespace

template <int D, bool BLOCKS>
flex_status_t fwd_dispatch(flex_dtype_t dtype, int score, int mask, const CUtensorMap& mq, const CUtensorMap& mk,
                           const CUtensorMap& mv, const FwdParams& p, int n_units, cudaStream_t s) {
  if (dtype == FLEX_DTYPE_BF16) return dispatch_score<D, __nv_bfloat16, BLOCKS>(score, mask, mq, mk, mv, p, n_units, s);
  return dispatch_score<D, __half, BLOCKS>(score, mask, mq, mk, mv, p, n_units, s);
}

}  // namespace flexattn
