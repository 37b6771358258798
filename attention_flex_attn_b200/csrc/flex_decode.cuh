// flex_decode.cuh -- decode attention: one query row per (batch, head) against a KV cache
// whose valid length differs per sequence (IREE issue 19015 "[ROCM] Support dynamic
// key-value cache sequence length", example IR: q [B,H,1,D], K/V [B,H,?,D], an f16
// additive mask [B,H,1,?], f32 accumulation).
//
// Split-KV ("flash decoding"): the cache of each (b, kv head) is cut into chunks of
// CH positions (128 or 256, a run-time choice between two instantiations).
// decode_split_kernel handles one chunk for GT query heads that share a kv head: it streams the chunk's K rows with 16-byte read-only loads, forms the scores
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
#include <type_traits>

#include "ptx_sm100.cuh"

namespace flexattn {

constexpr int kChunkMin = 128;        // cache positions per split: the two sizes built
constexpr int kChunkMax = 256;
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
  int B, H, Hkv, G, cap, split, n_splits;  // split: positions per chunk (CH of the kernels)
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

template <int D, typename T, int GT, int CH>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecodeParams p) {
  constexpr int LPR = D / 8;            // lanes per cache row (8 elements = 16 bytes each)
  constexpr int RPW = 32 / LPR;         // rows per warp per load instruction
  constexpr int ROWS_PER_PASS = kDecWarps * RPW;
  constexpr int U = 8;                  // loads in flight per lane

  __shared__ float s_sc[GT][CH];
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
  const int j0 = split * CH;
  if (L <= 0 || j0 >= L) return;
  const int n = min(CH, L - j0);

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
  for (int base = 0; base < CH; base += ROWS_PER_PASS * U) {
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
        if (sub == 0 && row < CH) s_sc[g][row] = acc;
      }
    }
  }
  __syncthreads();

  // ---- chunk-local softmax per head (mask added after the scale, in base 2)
  for (int g = warp; g < GT; g += kDecWarps) {
    const T* mrow = p.mask ? reinterpret_cast<const T*>(p.mask) + (static_cast<int64_t>(b) * p.H + h0 + g) * p.cap + j0
                           : nullptr;
    float vals[CH / 32];
    float mx = -INFINITY;
#pragma unroll
    for (int t = 0; t < CH / 32; ++t) {
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
    for (int t = 0; t < CH / 32; ++t) {
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
  for (int base = 0; base < CH; base += ROWS_PER_PASS * U) {
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

// ---------------------------------------------------------------------------------
// Grouped-query decode (G = H / Hkv >= 2): the G query heads of one kv head share every
// K/V byte, so the per-byte arithmetic grows with G.  This kernel puts up to 16 heads in
// the 16 rows of warp-level tensor-core MMAs (mma.sync m16n8k16, fp32 accumulate), which
// makes the arithmetic per byte independent of G and leaves the kernel bound by HBM.
// Each warp owns CH / 4 keys (64 or 32) of the chunk:
//  * S = Q K^T: K rows are loaded straight into B fragments, 16 bytes per lane.  Within
//    each 32-wide slice of the head dimension the contraction index is permuted the same
//    way in the Q (A) and K (B) fragments, so each lane reads 8 consecutive elements.
//  * the warp-local softmax works on the accumulator fragments; P is repacked in
//    registers as the A fragment of P V (the accumulator layout of S over two 8-key
//    tiles is the A layout of one 16-key step).
//  * V rows are loaded 16 bytes per lane and transposed in registers with movmatrix into
//    B fragments; this permutes the head dimension of O, which is undone on the store.
// The four warps' partial results are merged through shared memory into one (O, LSE)
// partial per chunk, in the same workspace format as decode_split_kernel.
constexpr int kGqaRows = 16;

template <typename T>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

__device__ __forceinline__ uint32_t transpose8x8(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

template <typename T>
__device__ __forceinline__ uint32_t pack_pair(float lo, float hi) {
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}

__device__ __forceinline__ uint32_t u4_at(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

template <int D, typename T, int CH>
__global__ void __launch_bounds__(kDecThreads, 4) decode_gqa_kernel(const DecodeParams p) {
  constexpr int KC = D / 32;  // 32-wide slices of the head dimension
  constexpr int KPW = CH / kDecWarps;  // keys per warp
  constexpr int NT = KPW / 8;          // 8-key tiles of S per warp
  constexpr int KS = KPW / 16;         // 16-key steps of P V per warp
  static_assert(NT % 2 == 0 && KS >= 1, "chunk too small for the warp tiling");
  __shared__ float s_m[kDecWarps][kGqaRows], s_l[kDecWarps][kGqaRows];
  __shared__ __align__(16) float s_o[kDecWarps][kGqaRows][D];

  const int split = blockIdx.x;
  const int ngrp = (p.G + kGqaRows - 1) / kGqaRows;
  const int grp = blockIdx.y % ngrp;
  const int bk = blockIdx.y / ngrp;
  const int hkv = bk % p.Hkv;
  const int b = bk / p.Hkv;
  const int h0 = hkv * p.G + grp * kGqaRows;
  const int gt = min(kGqaRows, p.G - grp * kGqaRows);  // valid MMA rows (query heads)

  const int L = checked_len(p, b);
  const int j0 = split * CH;
  if (L <= 0 || j0 >= L) return;
  const int n = min(CH, L - j0);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int kw0 = warp * KPW;
  const T* kbase = reinterpret_cast<const T*>(p.k) + ((static_cast<int64_t>(b) * p.Hkv + hkv) * p.cap + j0) * D;
  const T* vbase = reinterpret_cast<const T*>(p.v) + ((static_cast<int64_t>(b) * p.Hkv + hkv) * p.cap + j0) * D;

  // Q fragments: rows g and g + 8, head-dimension elements 32c + 8q .. 32c + 8q + 7.
  uint4 qa[KC][2];
#pragma unroll
  for (int c = 0; c < KC; ++c)
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = g + 8 * hr;
      qa[c][hr] = row < gt ? *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(p.q) +
                                                             (static_cast<int64_t>(b) * p.H + h0 + row) * D + 32 * c + 8 * q)
                           : make_uint4(0, 0, 0, 0);
    }

  // ---- S = Q K^T over this warp's KPW keys (NT tiles of 8 keys)
  float sc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; nt += 2) {
    uint4 kr[2][KC];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int key = kw0 + (nt + t) * 8 + g;
#pragma unroll
      for (int c = 0; c < KC; ++c)
        kr[t][c] = key < n ? ldg_nc_v4(kbase + static_cast<int64_t>(key) * D + 32 * c + 8 * q) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int c = 0; c < KC; ++c)
#pragma unroll
        for (int sub = 0; sub < 2; ++sub) {
          const uint32_t a[4] = {u4_at(qa[c][0], 2 * sub), u4_at(qa[c][1], 2 * sub), u4_at(qa[c][0], 2 * sub + 1),
                                 u4_at(qa[c][1], 2 * sub + 1)};
          mma16816<T>(acc, a, u4_at(kr[t][c], 2 * sub), u4_at(kr[t][c], 2 * sub + 1));
        }
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt + t][e] = acc[e];
    }
  }

  // ---- scale (base 2), padding, additive mask; warp-local softmax per row
  const T* mrow0 = nullptr;
  const T* mrow1 = nullptr;
  if (p.mask != nullptr) {
    if (g < gt) mrow0 = reinterpret_cast<const T*>(p.mask) + (static_cast<int64_t>(b) * p.H + h0 + g) * p.cap + j0;
    if (g + 8 < gt) mrow1 = reinterpret_cast<const T*>(p.mask) + (static_cast<int64_t>(b) * p.H + h0 + g + 8) * p.cap + j0;
  }
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = kw0 + nt * 8 + 2 * q + (e & 1);
      const bool upper = e >= 2;
      const int row = g + 8 * (upper ? 1 : 0);
      float x = -INFINITY;
      if (key < n && row < gt) {
        x = sc[nt][e] * p.scale_log2;
        const T* mr = upper ? mrow1 : mrow0;
        if (mr) x += to_float(mr[key]) * kDecLog2e;
      }
      sc[nt][e] = x;
      if (upper) m1 = fmaxf(m1, x);
      else m0 = fmaxf(m0, x);
    }
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
  }
  const float ms0 = m0 == -INFINITY ? 0.f : m0, ms1 = m1 == -INFINITY ? 0.f : m1;
  float l0 = 0.f, l1 = 0.f;
  uint32_t pa[KS][4];  // A fragments of P for the KS 16-key steps
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const float p0 = ex2_approx(sc[nt][0] - ms0), p1 = ex2_approx(sc[nt][1] - ms0);
    const float p2 = ex2_approx(sc[nt][2] - ms1), p3 = ex2_approx(sc[nt][3] - ms1);
    l0 += p0 + p1;
    l1 += p2 + p3;
    pa[nt >> 1][(nt & 1) * 2 + 0] = pack_pair<T>(p0, p1);
    pa[nt >> 1][(nt & 1) * 2 + 1] = pack_pair<T>(p2, p3);
  }
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }

  // ---- O = P V: per 16-key step and 32-wide slice, two 16-byte loads and 8 transposes
  float o[KC][4][4];
#pragma unroll
  for (int c = 0; c < KC; ++c)
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[c][r][e] = 0.f;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int keyA = kw0 + 16 * ks + g, keyB = keyA + 8;
    uint4 va[KC], vb[KC];
#pragma unroll
    for (int c = 0; c < KC; ++c) {
      va[c] = keyA < n ? ldg_nc_v4(vbase + static_cast<int64_t>(keyA) * D + 32 * c + 8 * q) : make_uint4(0, 0, 0, 0);
      vb[c] = keyB < n ? ldg_nc_v4(vbase + static_cast<int64_t>(keyB) * D + 32 * c + 8 * q) : make_uint4(0, 0, 0, 0);
    }
    // A fragment rows g / g+8, k = 2q, 2q+1 (keys 16ks + 2q..) and 2q+8, 2q+9 (keys 16ks + 8 + 2q..)
    const uint32_t a[4] = {pa[ks][0], pa[ks][1], pa[ks][2], pa[ks][3]};
#pragma unroll
    for (int c = 0; c < KC; ++c)
#pragma unroll
      for (int r = 0; r < 4; ++r)
        mma16816<T>(o[c][r], a, transpose8x8(u4_at(va[c], r)), transpose8x8(u4_at(vb[c], r)));
  }

  // ---- merge the four warps (each relative to its own row max) into one chunk partial
  if (q == 0) {
    s_m[warp][g] = m0;
    s_m[warp][g + 8] = m1;
    s_l[warp][g] = l0;
    s_l[warp][g + 8] = l1;
  }
  // o[c][r][0..1] hold rows g, o[c][r][2..3] row g + 8, head-dim 32c + 8q + 2r + {0, 1}
#pragma unroll
  for (int c = 0; c < KC; ++c)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int d = 32 * c + 8 * q + 2 * r;
      *reinterpret_cast<float2*>(&s_o[warp][g][d]) = make_float2(o[c][r][0], o[c][r][1]);
      *reinterpret_cast<float2*>(&s_o[warp][g + 8][d]) = make_float2(o[c][r][2], o[c][r][3]);
    }
  __syncthreads();
  for (int idx = threadIdx.x; idx < gt * D; idx += kDecThreads) {
    const int row = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, s_m[w][row]);
    float acc = 0.f, wsum = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) {
        const float mw = s_m[w][row];
        if (mw == -INFINITY) continue;
        const float f = ex2_approx(mw - M);
        wsum = fmaf(f, s_l[w][row], wsum);
        acc = fmaf(f, s_o[w][row][d], acc);
      }
    }
    const int64_t grow = static_cast<int64_t>(b) * p.H + h0 + row;
    p.part_o[(grow * p.n_splits + split) * D + d] = wsum > 0.f ? acc / wsum : 0.f;
    if (d == 0) p.part_lse[grow * p.n_splits + split] = wsum > 0.f ? M + lg2_approx(wsum) : -INFINITY;
  }
}

// One warp per (b, h) row: merge the chunks written by the split kernels.  Lane s holds the
// log-sum-exp of chunk s (chunks beyond 32 are folded in a second round), the weights
// 2^(lse_s - lse) are broadcast by shuffle, and the partial outputs of eight chunks are
// loaded at a time so their latencies overlap.
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
  const int ns = (L + p.split - 1) / p.split;
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
    for (int s0 = 0; s0 < ns; s0 += 32) {
      // weight of chunk s0 + lane (0 for empty or missing chunks)
      const int sl = s0 + lane;
      const float ls = sl < ns ? plse[sl] : -INFINITY;
      const float wl = ls == -INFINITY ? 0.f : ex2_approx(ls - M);
      float wsum = wl;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
      W += wsum;
      const int cnt = min(32, ns - s0);
      const float* po = p.part_o + (static_cast<int64_t>(row) * p.n_splits + s0) * D + lane * PER;
      for (int t0 = 0; t0 < cnt; t0 += 8) {
        float v[8][PER];
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
          for (int e = 0; e < PER; ++e) v[t][e] = t0 + t < cnt ? po[(t0 + t) * D + e] : 0.f;
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const float w = __shfl_sync(0xffffffffu, wl, (t0 + t) & 31);
#pragma unroll
          for (int e = 0; e < PER; ++e) o[e] = fmaf(w, v[t][e], o[e]);
        }
      }
    }
  }
  T* out = reinterpret_cast<T*>(p.o) + static_cast<int64_t>(row) * D + lane * PER;
  const float inv = W > 0.f ? 1.0f / W : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) store_out(out + e, o[e] * inv);
  if (lane == 0 && p.lse != nullptr) p.lse[row] = W > 0.f ? (M + lg2_approx(W)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace flexattn
