// flex_decode_launch.cu -- launches of the split-KV decode kernels and their combine:
// one query head per kv head runs the CUDA-core kernel, grouped heads the tensor-core
// kernel, whose work per byte of cache does not grow with the group size.
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

template <int D, typename T, int CH>
flex_status_t decode_by_group(const DecodeParams& p, cudaStream_t s) {
  if (p.G >= 2) return launch_decode_gqa<D, T, CH>(p, s);
  return launch_decode<D, T, 1, CH>(p, s);
}

template <int D, typename T>
flex_status_t decode_by_split(const DecodeParams& p, cudaStream_t s) {
  if (p.split == kChunkMin) return decode_by_group<D, T, kChunkMin>(p, s);
  return decode_by_group<D, T, kChunkMax>(p, s);
}

}  // namespace

flex_status_t decode_dispatch(int D, flex_dtype_t dtype, const DecodeParams& p, cudaStream_t s) {
  if (D == 128)
    return dtype == FLEX_DTYPE_BF16 ? decode_by_split<128, __nv_bfloat16>(p, s) : decode_by_split<128, __half>(p, s);
  return dtype == FLEX_DTYPE_BF16 ? decode_by_split<64, __nv_bfloat16>(p, s) : decode_by_split<64, __half>(p, s);
}

}  // namespace flexattn
