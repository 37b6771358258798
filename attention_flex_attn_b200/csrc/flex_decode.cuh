// flex_decode.cuh -- decode attention: one query row per (batch, head) against a KV cache
// whose valid length differs per sequence (IREE issue 19015 "[ROCM] Support dynamic
// key-value cache sequence length", example IR: q [B,H,1,D], K/V [B,H,?,D], an f16
// additive mask [B,H,1,?], f32 accumulation).
//
// Split-KV ("flash decoding"): the cache of each (b, kv head) is cut into chunks of
// kChunk positions.  decode_split_kernel handles one chunk for GT query heads that share
// a kv head: it streams the chunk's K rows with 16-byte read-only loads, forms the scores
// (scale * q.k + mask) in base 2, takes the chunk-local softmax and streams V for
// sum_j p_j V_j.  Each chunk writes its normalised partial output and its base-2
// log-sum-exp to the workspace.  decode_combine_kernel merges the chunks of each
// (b, h) row: lse = log2 sum_s 2^lse_s, O = sum_s 2^(lse_s - lse) o_s.
// kv_len is read on the device, so no host synchronisation is needed; chunks that start
// at or beyond kv_len[b] exit at once.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "ptx_sm100.cuh"

namespace flexattn {

constexpr int kChunk = 256;           // cache positions per split
constexpr int kDecThreads = 128;
constexpr int kDecWarps = kDecThreads / 32;
constexpr unsigned kStatusBadKvLen = 1u;
constexpr float kDecLog2e = 1.4426950408889634f;

struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  const int32_t* kv_len;
  const void* mask;   // [B, H, 1, cap] or nullptr
  void* o;
  float* lse;
  float* part_o;      // [B*H, n_splits, D]
  float* part_lse;    // [B*H, n_splits]
  unsigned* status;
  int B, H, Hkv, G, cap, n_splits;
  float scale_log2;
};

template <typename T>
__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]);
template <>
__device__ __forceinline__ void unpack8<__half>(const uint4& u, float (&f)[8]) {
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
template <>
__device__ __forceinline__ void unpack8<__nv_bfloat16>(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ float to_float(__half x) { return __half2float(x); }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store_out(__half* p, float x) { *p = __float2half_rn(x); }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

__device__ __forceinline__ uint4 ldg_nc_v4(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

__device__ __forceinline__ int checked_len(const DecodeParams& p, int b) {
  const int L = p.kv_len[b];
  return (L < 0 || L > p.cap) ? -1 : L;
}

template <int D, typename T, int GT>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecodeParams p) {
  constexpr int LPR = D / 8;            // lanes per cache row (8 elements = 16 bytes each)
  constexpr int RPW = 32 / LPR;         // rows per warp per load instruction
  constexpr int ROWS_PER_PASS = kDecWarps * RPW;
  constexpr int U = 8;                  // loads in flight per lane

  __shared__ float s_sc[GT][kChunk];
  __shared__ float s_red[kDecWarps][GT][D];
  __shared__ float s_m[GT], s_l[GT];

  const int split = blockIdx.x;
  const int ngt = p.G / GT;
  const int gt = blockIdx.y % ngt;
  const int bk = blockIdx.y / ngt;
  const int hkv = bk % p.Hkv;
  const int b = bk / p.Hkv;
  const int h0 = hkv * p.G + gt * GT;

  const int L = checked_len(p, b);
  const int j0 = split * kChunk;
  if (L <= 0 || j0 >= L) return;
  const int n = min(kChunk, L - j0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = lane % LPR, rsub = lane / LPR;

  const T* kbase = reinterpret_cast<const T*>(p.k) + ((static_cast<int64_t>(b) * p.Hkv + hkv) * p.cap + j0) * D;
  const T* vbase = reinterpret_cast<const T*>(p.v) + ((static_cast<int64_t>(b) * p.Hkv + hkv) * p.cap + j0) * D;

  float qf[GT][8];
#pragma unroll
  for (int g = 0; g < GT; ++g) {
    const T* qrow = reinterpret_cast<const T*>(p.q) + (static_cast<int64_t>(b) * p.H + h0 + g) * D + 8 * sub;
    const uint4 u = *reinterpret_cast<const uint4*>(qrow);
    unpack8<T>(u, qf[g]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] *= p.scale_log2;
  }

  // ---- scores: s = scale*log2(e) * q.k over the chunk
  for (int base = 0; base < kChunk; base += ROWS_PER_PASS * U) {
    uint4 kr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * ROWS_PER_PASS + warp * RPW + rsub;
      kr[u] = row < n ? ldg_nc_v4(kbase + static_cast<int64_t>(row) * D + 8 * sub) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * ROWS_PER_PASS + warp * RPW + rsub;
      float kf[8];
      unpack8<T>(kr[u], kf);
#pragma unroll
      for (int g = 0; g < GT; ++g) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(qf[g][e], kf[e], acc);
#pragma unroll
        for (int off = LPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (sub == 0 && row < kChunk) s_sc[g][row] = acc;
      }
    }
  }
  __syncthreads();

  // ---- chunk-local softmax per head (mask added after the scale, in base 2)
  for (int g = warp; g < GT; g += kDecWarps) {
    const T* mrow = p.mask ? reinterpret_cast<const T*>(p.mask) + (static_cast<int64_t>(b) * p.H + h0 + g) * p.cap + j0
                           : nullptr;
    float vals[kChunk / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < kChunk / 32; ++t) {
      const int e = lane + 32 * t;
      float x = -INFINITY;
      if (e < n) {
        x = s_sc[g][e];
        if (mrow) x += to_float(mrow[e]) * kDecLog2e;
      }
      vals[t] = x;
      mx = fmaxf(mx, x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float ms = mx == -INFINITY ? 0.f : mx;
    float sum = 0.f;
#pragma unroll
    for (int t = 0; t < kChunk / 32; ++t) {
      const float e2 = ex2_approx(vals[t] - ms);
      s_sc[g][lane + 32 * t] = e2;
      sum += e2;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane == 0) {
      s_m[g] = mx;
      s_l[g] = sum;
    }
  }
  __syncthreads();

  // ---- o = sum_j p_j V_j over the chunk
  float acc[GT][8];
#pragma unroll
  for (int g = 0; g < GT; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  for (int base = 0; base < kChunk; base += ROWS_PER_PASS * U) {
    uint4 vr[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * ROWS_PER_PASS + warp * RPW + rsub;
      vr[u] = row < n ? ldg_nc_v4(vbase + static_cast<int64_t>(row) * D + 8 * sub) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = base + u * ROWS_PER_PASS + warp * RPW + rsub;
      if (row < n) {
        float vf[8];
        unpack8<T>(vr[u], vf);
#pragma unroll
        for (int g = 0; g < GT; ++g) {
          const float pg = s_sc[g][row];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < GT; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float x = acc[g][e];
#pragma unroll
      for (int off = LPR; off < 32; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
      acc[g][e] = x;
    }
  if (rsub == 0) {
#pragma unroll
    for (int g = 0; g < GT; ++g)
#pragma unroll
      for (int e = 0; e < 8; ++e) s_red[warp][g][8 * sub + e] = acc[g][e];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < GT * D; idx += kDecThreads) {
    const int g = idx / D, d = idx % D;
    float x = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) x += s_red[w][g][d];
    const float l = s_l[g];
    const int64_t row = static_cast<int64_t>(b) * p.H + h0 + g;
    p.part_o[(row * p.n_splits + split) * D + d] = l > 0.f ? x / l : 0.f;
    if (d == 0) p.part_lse[row * p.n_splits + split] = l > 0.f ? s_m[g] + lg2_approx(l) : -INFINITY;
  }
}

// One warp per (b, h) row: merge the chunks written by decode_split_kernel.
template <int D, typename T>
__global__ void __launch_bounds__(kDecThreads) decode_combine_kernel(const DecodeParams p) {
  constexpr int PER = D / 32;
  const int row = blockIdx.x * kDecWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.B * p.H) return;
  const int b = row / p.H;
  int L = checked_len(p, b);
  if (L < 0) {
    if (lane == 0 && row % p.H == 0) atomicOr(p.status, kStatusBadKvLen);
    L = 0;
  }
  const int ns = (L + kChunk - 1) / kChunk;
  const float* plse = p.part_lse + static_cast<int64_t>(row) * p.n_splits;
  float M = -INFINITY;
  for (int s = lane; s < ns; s += 32) M = fmaxf(M, plse[s]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
  float W = 0.f;
  if (M != -INFINITY) {
    for (int s = 0; s < ns; ++s) {
      const float ls = plse[s];
      if (ls == -INFINITY) continue;
      const float w = ex2_approx(ls - M);
      W += w;
      const float* po = p.part_o + (static_cast<int64_t>(row) * p.n_splits + s) * D + lane * PER;
#pragma unroll
      for (int e = 0; e < PER; ++e) o[e] = fmaf(w, po[e], o[e]);
    }
  }
  T* out = reinterpret_cast<T*>(p.o) + static_cast<int64_t>(row) * D + lane * PER;
  const float inv = W > 0.f ? 1.0f / W : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) store_out(out + e, o[e] * inv);
  if (lane == 0 && p.lse != nullptr) p.lse[row] = W > 0.f ? (M + lg2_approx(W)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace flexattn
