// flex_fwd_inst.cuh -- body of the forward instantiation units: sets the shared-memory
// attribute once per kernel and device, and dispatches (dtype, score_mod, mask_mod)
// onto the compile-time specialised kernels.  Included by flex_fwd_d*.cu only, each of
// which instantiates fwd_dispatch for one (head dim, block mask) pair, or the persistent
// launches for one head dim (FLEX_FWD_PERSISTENT_UNIT defined).
#pragma once

#include <atomic>
#include <cstdint>

#include "launch.cuh"

namespace flexattn {
namespace {

// The analytic masks without documents can run on the persistent kernel: one CTA per SM
// walking its units back to back, the K/V stream running on from one unit to the next.
// The host picks it (FwdParams::persist_grid > 0) when the units are short, and for
// causal-like masks only while all K/V fit in L2 (their units, sorted heaviest first,
// spread over the CTAs in snake order).  Block and document masks keep per-unit bitmaps.
template <int MASK, bool BLOCKS>
constexpr bool fwd_persistable() {
  return !BLOCKS && (MASK == kMaskNone || MASK == kMaskSliding || MASK == kMaskCausal || MASK == kMaskOffset);
}

// Per-device "attribute already set" bits, one set per kernel instantiation (the tag
// parameters make every instantiation own its static).
template <int D, typename T, int SCORE, int MASK, bool BLOCKS, bool PERSIST, typename K>
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

}  // namespace

// The persistent kernels, instantiated in flex_fwd_d*_persist.cu.
template <int D, typename T, int SCORE, int MASK>
flex_status_t launch_fwd_persistent(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                    const FwdParams& p, cudaStream_t stream);

namespace {

template <int D, typename T, int SCORE, int MASK, bool BLOCKS>
flex_status_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const FwdParams& p,
                         int n_units, cudaStream_t stream) {
  if constexpr (fwd_persistable<MASK, BLOCKS>()) {
    if (p.persist_grid > 0) return launch_fwd_persistent<D, T, SCORE, MASK>(mq, mk, mv, p, stream);
  }
  auto kern = flex_fwd_kernel<D, T, SCORE, MASK, BLOCKS, false>;
  constexpr int kSmem = FwdSmem<D, BLOCKS, is_doc_mask(MASK)>::kAlloc;
  if (!ensure_smem_attr<D, T, SCORE, MASK, BLOCKS, false>(kern, kSmem)) return FLEX_ERR_CUDA;
  kern<<<p.n_items, kFwdThreads, kSmem, stream>>>(mq, mk, mv, p);
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

#ifdef FLEX_FWD_PERSISTENT_UNIT
template <int D, typename T, int SCORE, int MASK>
flex_status_t launch_fwd_persistent(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                    const FwdParams& p, cudaStream_t stream) {
  static_assert(fwd_persistable<MASK, false>(), "no persistent kernel for this mask");
  auto kern = flex_fwd_kernel<D, T, SCORE, MASK, false, true>;
  constexpr int kSmem = FwdSmem<D, false, false>::kAlloc;
  if (!ensure_smem_attr<D, T, SCORE, MASK, false, true>(kern, kSmem)) return FLEX_ERR_CUDA;
  kern<<<p.persist_grid, kFwdThreads, kSmem, stream>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

// every (dtype, score_mod, mask) of head dim D that fwd_dispatch may send to the persistent kernel
#define FLEX_FWD_PERSISTENT_INSTANCES(D) \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreNone, kMaskNone>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreNone, kMaskSliding>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreNone, kMaskCausal>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreNone, kMaskOffset>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreAlibi, kMaskNone>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreAlibi, kMaskSliding>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreAlibi, kMaskCausal>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __half, kScoreAlibi, kMaskOffset>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreNone, kMaskNone>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreNone, kMaskSliding>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreNone, kMaskCausal>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreNone, kMaskOffset>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreAlibi, kMaskNone>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreAlibi, kMaskSliding>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreAlibi, kMaskCausal>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t); \
  template flex_status_t launch_fwd_persistent<D, __nv_bfloat16, kScoreAlibi, kMaskOffset>( \
      const CUtensorMap&, const CUtensorMap&, const CUtensorMap&, const FwdParams&, cudaStream_t);
#endif

}  // namespace flexattn
