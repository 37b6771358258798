// flex_fwd_fp8.cu -- launches of the 8-bit forward: the V transpose, then the kernel
// instantiation for (score_mod, mask_mod, block mask or not).
#include <atomic>

#include "flex_fwd_fp8_sm100.cuh"
#include "launch.cuh"

namespace flexattn {
namespace {

template <int SCORE, int MASK, bool BLOCKS>
flex_status_t launch_fp8(const Fp8Maps& m, const Fp8Params& p, int n_units, cudaStream_t s) {
  static std::atomic<uint64_t> done{0};
  auto kern = flex_fwd_fp8_kernel<SCORE, MASK, BLOCKS>;
  constexpr int kSmem = Fp8Smem<BLOCKS, is_doc_mask(MASK)>::kAlloc;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLEX_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(done.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem) != cudaSuccess)
      return FLEX_ERR_CUDA;
    done.fetch_or(bit, std::memory_order_acq_rel);
  }
  kern<<<n_units, kFwdThreads, kSmem, s>>>(m.q, m.k, m.vt, p);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

template <int SCORE, bool BLOCKS>
flex_status_t fp8_mask(int mask, const Fp8Maps& m, const Fp8Params& p, int n_units, cudaStream_t s) {
  switch (mask) {
    case kMaskNone: return launch_fp8<SCORE, kMaskNone, BLOCKS>(m, p, n_units, s);
    case kMaskCausal: return launch_fp8<SCORE, kMaskCausal, BLOCKS>(m, p, n_units, s);
    case kMaskSliding: return launch_fp8<SCORE, kMaskSliding, BLOCKS>(m, p, n_units, s);
    case kMaskOffset: return launch_fp8<SCORE, kMaskOffset, BLOCKS>(m, p, n_units, s);
    case kMaskDocument: return launch_fp8<SCORE, kMaskDocument, BLOCKS>(m, p, n_units, s);
    case kMaskDocumentCausal: return launch_fp8<SCORE, kMaskDocumentCausal, BLOCKS>(m, p, n_units, s);
  }
  return FLEX_ERR_UNSUPPORTED;
}

template <bool BLOCKS>
flex_status_t fp8_score(int score, int mask, const Fp8Maps& m, const Fp8Params& p, int n_units, cudaStream_t s) {
  if (score == kScoreNone) return fp8_mask<kScoreNone, BLOCKS>(mask, m, p, n_units, s);
  return fp8_mask<kScoreAlibi, BLOCKS>(mask, m, p, n_units, s);
}

}  // namespace

flex_status_t fp8_dispatch(int score, int mask, bool blocks, const uint8_t* v, uint8_t* vt, int64_t kv_rows,
                           const Fp8Maps& m, const Fp8Params& p, int n_units, cudaStream_t s) {
  const int n_tiles = p.Skv_pad / 128;
  if (p.D == 128)
    fp8_transpose_v_kernel<128><<<static_cast<unsigned>(kv_rows * n_tiles), 256, 0, s>>>(v, vt, p.Skv, p.Skv_pad, n_tiles);
  else
    fp8_transpose_v_kernel<64><<<static_cast<unsigned>(kv_rows * n_tiles), 256, 0, s>>>(v, vt, p.Skv, p.Skv_pad, n_tiles);
  if (cudaGetLastError() != cudaSuccess) return FLEX_ERR_CUDA;
  return blocks ? fp8_score<true>(score, mask, m, p, n_units, s) : fp8_score<false>(score, mask, m, p, n_units, s);
}

}  // namespace flexattn
