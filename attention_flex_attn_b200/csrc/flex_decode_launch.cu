// flex_decode_launch.cu -- launches of the split-KV decode kernels and their combine:
// one query head per kv head runs the CUDA-core kernel, grouped heads the tensor-core
// kernel, whose work per byte of cache does not grow with the group size.
#include <atomic>

#include "launch.cuh"

namespace flexattn {
namespace {

template <int D, typename T, int GT, int CH>
flex_status_t launch_decode(const DecodeParams& p, cudaStream_t s) {
  dim3 grid(p.n_splits, p.B * p.Hkv * (p.G / GT));
  decode_split_kernel<D, T, GT, CH><<<grid, kDecThreads, 0, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FLEX_ERR_CUDA;
  const int rows = p.B * p.H;
  decode_combine_kernel<D, T><<<(rows + kDecWarps - 1) / kDecWarps, kDecThreads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

template <int D, typename T, int CH>
flex_status_t launch_decode_gqa(const DecodeParams& p, cudaStream_t s) {
  dim3 grid(p.n_splits, p.B * p.Hkv * ((p.G + kGqaRows - 1) / kGqaRows));
  decode_gqa_kernel<D, T, CH><<<grid, kDecThreads, 0, s>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FLEX_ERR_CUDA;
  const int rows = p.B * p.H;
  decode_combine_kernel<D, T><<<(rows + kDecWarps - 1) / kDecWarps, kDecThreads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

// Grouped heads, persistent TMA-fed kernel: one CTA per SM, the chunk list built on the
// device from kv_len.
template <int D, typename T>
flex_status_t launch_decode_gqa_tma(const DecodeParams& p, const DecodeMaps& m, cudaStream_t s) {
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FLEX_ERR_CUDA;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    if (cudaFuncSetAttribute(decode_gqa_tma_kernel<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             DtSmem<D>::kAlloc) != cudaSuccess)
      return FLEX_ERR_CUDA;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  decode_gqa_tma_kernel<D, T><<<m.grid, kDtThreads, DtSmem<D>::kAlloc, s>>>(m.k, m.v, m.m, p, m.mask_rows);
  if (cudaGetLastError() != cudaSuccess) return FLEX_ERR_CUDA;
  const int rows = p.B * p.H;
  decode_combine_kernel<D, T><<<(rows + kDecWarps - 1) / kDecWarps, kDecThreads, 0, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

template <int D, typename T, int CH>
flex_status_t decode_by_group(const DecodeParams& p, const DecodeMaps* m, cudaStream_t s) {
#ifndef FLEX_DECODE_GQA_REGISTERS
  if (p.G >= 2 && m != nullptr) return launch_decode_gqa_tma<D, T>(p, *m, s);
#endif
  if (p.G >= 2) return launch_decode_gqa<D, T, CH>(p, s);
  return launch_decode<D, T, 1, CH>(p, s);
}

template <int D, typename T>
flex_status_t decode_by_split(const DecodeParams& p, const DecodeMaps* m, cudaStream_t s) {
  if (p.split == kChunkMin) return decode_by_group<D, T, kChunkMin>(p, m, s);
  return decode_by_group<D, T, kChunkMax>(p, m, s);
}

}  // namespace

flex_status_t decode_dispatch(int D, flex_dtype_t dtype, const DecodeParams& p, const DecodeMaps* m,
                              cudaStream_t s) {
  if (D == 128)
    return dtype == FLEX_DTYPE_BF16 ? decode_by_split<128, __nv_bfloat16>(p, m, s)
                                    : decode_by_split<128, __half>(p, m, s);
  return dtype == FLEX_DTYPE_BF16 ? decode_by_split<64, __nv_bfloat16>(p, m, s) : decode_by_split<64, __half>(p, m, s);
}

}  // namespace flexattn
