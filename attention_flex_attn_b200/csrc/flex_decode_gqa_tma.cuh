// flex_decode_gqa_tma.cuh -- grouped-query decode (G = H / Hkv >= 2) as a persistent,
// warp-specialised kernel (IREE issue 19015 "[ROCM] Support dynamic key-value cache
// sequence length", example IR: one query row per head against a KV cache of dynamic
// length, f16 additive mask, f32 accumulation).
//
// The work is the list of chunks (b, kv head, group of up to 16 query heads, chunk c of
// `split` positions below kv_len[b]).  Every CTA builds the same compact list from kv_len
// on the device (a prefix sum over the batch), so chunks past a sequence's length cost
// nothing, and takes chunks blockIdx.x, blockIdx.x + gridDim.x, ... (one CTA per SM);
// consumer warp w takes the CTA's chunks w, w + 4, ...
//   warp 4      producer (one thread): streams the K and V tiles (64 positions each) of
//               every consumer's chunks with TMA (128-byte swizzle, positions past the
//               cache's capacity zero-filled), and with each K tile the additive mask's
//               [query heads x 64 positions] tile, into that consumer's own ring of slots,
//               polling the four rings so that a full one does not hold back the others;
//               12 x 16 KB per SM stay in flight, independent of the consumers' registers.
//   warps 0-3   consumers: per tile S = Q K^T with K fragments from ldmatrix (mma.sync
//               m16n8k16, the query heads in the MMA rows), scale + additive mask + online
//               softmax in registers, O += P V with V fragments from ldmatrix.trans; at the
//               end of a chunk the chunk's normalised partial output and base-2 LSE go to
//               the workspace in the format of decode_split_kernel, for
//               decode_combine_kernel.
// Each ring has one consumer, which uses its slots in the order the producer fills them,
// so a wait on a slot's full barrier never runs more than one phase ahead (a ring shared
// by the four consumers would let a consumer whose chunk lies two ring cycles ahead pass
// its parity wait on an earlier phase).  Every wait is bounded; on a timeout the kernel
// sets status bit 4 and all roles leave their loops.
#pragma once

#include <cuda.h>

#include "flex_decode.cuh"

namespace flexattn {

constexpr int kDtKeys = 64;                      // positions per K / V tile
constexpr int kDtConsumers = 4;                  // consumer warps
constexpr int kDtThreads = 32 * (kDtConsumers + 1);
constexpr int kDtProducerWarp = kDtConsumers;
constexpr unsigned kStatusDecTimeout = 4u;
constexpr int kDtMaxBatch = 1024;                // batch prefix sums kept in shared memory
constexpr uint64_t kDtWaitNs = 2000000000ull;

template <int D>
struct DtSmem {
  static constexpr int kBoxBytes = kDtKeys * 128;   // 64 rows x 64 16-bit elements
  static constexpr int kTileBytes = kDtKeys * D * 2;
  static constexpr int kMaskBytes = kGqaRows * kDtKeys * 2;  // mask tile: <= 16 heads x 64 positions
  static constexpr int kSlotBytes = kTileBytes + kMaskBytes;  // a multiple of 1024 (swizzle alignment)
  static constexpr int kSlots = D == 128 ? 12 : 20;   // kDtConsumers rings of kRing slots
  static constexpr int kRing = kSlots / kDtConsumers;
  static constexpr int kBarOff = kSlots * kSlotBytes;
  static constexpr int kFlagOff = kBarOff + 2 * kSlots * 8;
  static constexpr int kPrefOff = kFlagOff + 16;
  static constexpr int kBytes = kPrefOff + (kDtMaxBatch + 1) * 4;
  static constexpr int kAlloc = kBytes + 1024;      // slack to align the ring to 1024 bytes
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA exceeded");
  static_assert(kSlotBytes % 1024 == 0, "slots must keep the 1024-byte swizzle alignment");
};

// Non-blocking probe: has the phase with this parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.b32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Byte offset of the 16-byte piece holding elements [dim, dim + 8) of row `key` in a tile
// written by TMA as D / 64 boxes of [64 rows x 128 bytes] with the 128-byte swizzle.
__device__ __forceinline__ uint32_t dt_off(int key, int dim) {
  const int box = dim >> 6, chunk = (dim & 63) >> 3;
  return static_cast<uint32_t>(box * (kDtKeys * 128) + key * 128 + ((chunk ^ (key & 7)) << 4));
}

template <int D, typename T>
__global__ void __launch_bounds__(kDtThreads, 1)
    decode_gqa_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                          const __grid_constant__ CUtensorMap tmM, const DecodeParams p, int mask_rows) {
  using L = DtSmem<D>;
  constexpr int NS = L::kSlots;
  constexpr int NR = L::kRing;
  constexpr int KK = D / 16;   // k-steps of S
  constexpr int NO = D / 8;    // 8-wide column tiles of O
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_addr);
  auto bar_full = [&](int s) { return sbase + L::kBarOff + 8u * s; };
  auto bar_empty = [&](int s) { return sbase + L::kBarOff + 8u * (NS + s); };
  auto slot = [&](int s) { return sbase + static_cast<uint32_t>(s * L::kSlotBytes); };
  // the mask tile rides with the K tile: mask_rows (the group's query heads) x 64 positions,
  // streamed when mask_rows > 0, else read from global memory
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kFlagOff);
  int* pref = reinterpret_cast<int*>(sgen + L::kPrefOff);  // first chunk of each batch; pref[B] = total

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ngrp = (p.G + kGqaRows - 1) / kGqaRows;
  const int per_pos = p.Hkv * ngrp;  // chunks per chunk position of a sequence

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {  // exclusive prefix sum of the chunk counts over the batch
    int run = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
      const int b = b0 + lane;
      int cnt = 0;
      if (b < p.B) {
        const int Lb = checked_len(p, b);
        cnt = Lb > 0 ? (Lb + p.split - 1) / p.split * per_pos : 0;
      }
      int x = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
      }
      if (b < p.B) pref[b] = run + x - cnt;
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) pref[p.B] = run;
  }
  __syncthreads();
  const int total = pref[p.B];

  // chunk i -> (b, kv head, head group, chunk position); chunk positions vary fastest
  struct Chunk {
    int b, hkv, grp, c, len, ntiles;
  };
  auto chunk_of = [&](int i) {
    int lo = 0, hi = p.B - 1;  // last b with pref[b] <= i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pref[mid] <= i) lo = mid;
      else hi = mid - 1;
    }
    Chunk ch;
    ch.b = lo;
    const int r = i - pref[lo];
    const int npos = (pref[lo + 1] - pref[lo]) / per_pos;
    const int hg = r / npos;
    ch.c = r - hg * npos;
    ch.hkv = hg / ngrp;
    ch.grp = hg - ch.hkv * ngrp;
    const int Lb = checked_len(p, ch.b);
    ch.len = min(p.split, Lb - ch.c * p.split);
    ch.ntiles = (ch.len + kDtKeys - 1) / kDtKeys;
    return ch;
  };
  auto wait = [&](uint32_t bar, uint32_t parity) -> bool {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (!mbar_wait(bar, parity, p.status, kStatusDecTimeout, kDtWaitNs)) {
      *abort_flag = 1;
      return false;
    }
    return true;
  };

  if (warp == kDtProducerWarp) {
    // ============================================================ TMA producer
    if (lane == 0) {
      // per consumer w: its current chunk (ci >= total: done), the chunk's first row,
      // (b, kv head) row and tile count, the next load of it (two per tile: K, V) and the
      // ring position of that load
      int ci[kDtConsumers], y0[kDtConsumers], bk[kDtConsumers], nt[kDtConsumers], ld[kDtConsumers],
          rw[kDtConsumers], mh[kDtConsumers], mb[kDtConsumers];
#pragma unroll
      for (int w = 0; w < kDtConsumers; ++w) {
        ci[w] = blockIdx.x + w * gridDim.x;
        ld[w] = rw[w] = 0;
        nt[w] = y0[w] = bk[w] = mh[w] = mb[w] = 0;
        if (ci[w] < total) {
          const Chunk ch = chunk_of(ci[w]);
          y0[w] = ch.c * p.split;
          bk[w] = ch.b * p.Hkv + ch.hkv;
          nt[w] = ch.ntiles;
          mh[w] = ch.hkv * p.G + ch.grp * kGqaRows;
          mb[w] = ch.b;
        }
      }
      uint64_t t_last = global_timer_ns();
      bool ok = true;
      while (ok) {
        bool any = false, progressed = false;
#pragma unroll
        for (int w = 0; w < kDtConsumers; ++w) {
          if (ci[w] >= total) continue;
          any = true;
          const int s = w * NR + rw[w] % NR;
          if (rw[w] >= NR && !mbar_test(bar_empty(s), (static_cast<uint32_t>(rw[w] / NR) & 1u) ^ 1u)) continue;
          const bool with_mask = mask_rows > 0 && (ld[w] & 1) == 0;
          mbar_arrive_expect_tx(bar_full(s), L::kTileBytes + (with_mask ? mask_rows * kDtKeys * 2 : 0));
          const CUtensorMap* map = (ld[w] & 1) ? &tmV : &tmK;
#pragma unroll
          for (int box = 0; box < D / 64; ++box)
            tma_load_3d(slot(s) + box * L::kBoxBytes, map, bar_full(s), box * 64, y0[w] + (ld[w] >> 1) * kDtKeys,
                        bk[w]);
          if (with_mask)  // rows h0 .. h0 + mask_rows - 1 of batch b: [cap, H, B] map
            tma_load_3d(slot(s) + L::kTileBytes, &tmM, bar_full(s), y0[w] + (ld[w] >> 1) * kDtKeys, mh[w], mb[w]);
          ++rw[w];
          if (++ld[w] == 2 * nt[w]) {  // the chunk is streamed: the consumer's next one
            ci[w] += kDtConsumers * gridDim.x;
            ld[w] = 0;
            if (ci[w] < total) {
              const Chunk ch = chunk_of(ci[w]);
              y0[w] = ch.c * p.split;
              bk[w] = ch.b * p.Hkv + ch.hkv;
              nt[w] = ch.ntiles;
              mh[w] = ch.hkv * p.G + ch.grp * kGqaRows;
              mb[w] = ch.b;
            }
          }
          progressed = true;
        }
        if (!any) break;
        if (progressed) {
          t_last = global_timer_ns();
        } else if (*abort_flag || global_timer_ns() - t_last > kDtWaitNs) {
          if (!*abort_flag) atomicOr(p.status, kStatusDecTimeout);
          *abort_flag = 1;
          ok = false;
        }
      }
      // every issued copy must land before the CTA may exit
#pragma unroll
      for (int w = 0; w < kDtConsumers; ++w)
        for (int e = rw[w] - NR < 0 ? 0 : rw[w] - NR; e < rw[w]; ++e)
          mbar_wait(bar_full(w * NR + e % NR), static_cast<uint32_t>(e / NR) & 1u, p.status, kStatusDecTimeout,
                    kDtWaitNs);
    }
    return;
  }

  // ============================================================ consumer warps
  const int g = lane >> 2, q = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;  // ldmatrix: this lane's matrix and row
  int r = 0;  // position in this warp's ring of the next chunk's first load
  for (int i = blockIdx.x + warp * gridDim.x; i < total; i += kDtConsumers * gridDim.x) {
    const Chunk ch = chunk_of(i);
    const int r0 = r;
    r += 2 * ch.ntiles;
    const int h0 = ch.hkv * p.G + ch.grp * kGqaRows;
    const int gt = min(kGqaRows, p.G - ch.grp * kGqaRows);  // valid MMA rows (query heads)
    const bool row0 = g < gt, row1 = g + 8 < gt;
    const int j0 = ch.c * p.split;

    // Q fragments (A of S): rows g, g + 8; per k-step, elements 2q, 2q + 1 and 2q + 8, 2q + 9
    uint32_t qa[KK][4];
    {
      const uint32_t* q0p = reinterpret_cast<const uint32_t*>(reinterpret_cast<const T*>(p.q) +
                                                              (static_cast<int64_t>(ch.b) * p.H + h0 + g) * D);
      const uint32_t* q1p = q0p + 8 * D / 2;
#pragma unroll
      for (int kk = 0; kk < KK; ++kk) {
        qa[kk][0] = row0 ? q0p[kk * 8 + q] : 0u;
        qa[kk][1] = row1 ? q1p[kk * 8 + q] : 0u;
        qa[kk][2] = row0 ? q0p[kk * 8 + 4 + q] : 0u;
        qa[kk][3] = row1 ? q1p[kk * 8 + 4 + q] : 0u;
      }
    }
    const T* mrow0 = nullptr;
    const T* mrow1 = nullptr;
    if (p.mask != nullptr) {
      if (row0) mrow0 = reinterpret_cast<const T*>(p.mask) + (static_cast<int64_t>(ch.b) * p.H + h0 + g) * p.cap;
      if (row1) mrow1 = reinterpret_cast<const T*>(p.mask) + (static_cast<int64_t>(ch.b) * p.H + h0 + g + 8) * p.cap;
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[NO][4];
#pragma unroll
    for (int nt = 0; nt < NO; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
    bool ok = true;
    for (int t = 0; t < ch.ntiles && ok; ++t) {
      const int n = min(kDtKeys, ch.len - t * kDtKeys);  // valid positions of this tile
      const int key0 = j0 + t * kDtKeys;
      // additive mask of this lane's scores: from global memory (loaded before the tile's
      // data arrives) unless the producer streams it with the K tile
      float mk[8][4];
      if (mask_rows == 0) {
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = nt * 8 + 2 * q + (e & 1);
            const T* mr = e < 2 ? mrow0 : mrow1;
            mk[nt][e] = (mr != nullptr && key < n) ? to_float(mr[key0 + key]) * kDecLog2e : 0.f;
          }
      }
      // ---- S = Q K^T over the tile's 64 positions
      const int rK = r0 + 2 * t, sK = warp * NR + rK % NR;
      if (!wait(bar_full(sK), static_cast<uint32_t>(rK / NR) & 1u)) {
        ok = false;
        break;
      }
      if (mask_rows > 0) {  // rows g and g + 8 of the streamed mask tile ([rows][64] 16-bit)
        const T* mt = reinterpret_cast<const T*>(sgen + (sK * L::kSlotBytes + L::kTileBytes));
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int key = nt * 8 + 2 * q + (e & 1);
            const bool valid = e < 2 ? row0 : row1;
            mk[nt][e] = valid ? to_float(mt[(e < 2 ? g : g + 8) * kDtKeys + key]) * kDecLog2e : 0.f;
          }
      }
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = 0.f;
      const uint32_t kb = slot(sK);
#pragma unroll
      for (int kk = 0; kk < KK; ++kk)
#pragma unroll
        for (int nt = 0; nt < 8; nt += 2) {
          uint32_t b[4];  // b0, b1 of tile nt, then of tile nt + 1
          ldsm_x4(kb + dt_off((nt + (mi >> 1)) * 8 + rr, kk * 16 + (mi & 1) * 8), b);
          mma16816<T>(sc[nt], qa[kk], b[0], b[1]);
          mma16816<T>(sc[nt + 1], qa[kk], b[2], b[3]);
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(sK));  // K is in registers now
      // ---- scale (base 2), mask, valid positions; online softmax per row
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = nt * 8 + 2 * q + (e & 1);
          const bool upper = e >= 2;
          float x = -INFINITY;
          if (key < n && (upper ? row1 : row0)) x = fmaf(sc[nt][e], p.scale_log2, mk[nt][e]);
          sc[nt][e] = x;
          if (upper) mx1 = fmaxf(mx1, x);
          else mx0 = fmaxf(mx0, x);
        }
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
      const float a0 = m0 == -INFINITY ? 0.f : ex2_approx(m0 - n0);
      const float a1 = m1 == -INFINITY ? 0.f : ex2_approx(m1 - n1);
      m0 = n0;
      m1 = n1;
      const float ms0 = n0 == -INFINITY ? 0.f : n0, ms1 = n1 == -INFINITY ? 0.f : n1;
      float s0 = 0.f, s1 = 0.f;
      uint32_t pa[4][4];  // A fragments of P for the four 16-position steps
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p0 = ex2_approx(sc[nt][0] - ms0), p1 = ex2_approx(sc[nt][1] - ms0);
        const float p2 = ex2_approx(sc[nt][2] - ms1), p3 = ex2_approx(sc[nt][3] - ms1);
        s0 += p0 + p1;
        s1 += p2 + p3;
        pa[nt >> 1][(nt & 1) * 2 + 0] = pack_pair<T>(p0, p1);
        pa[nt >> 1][(nt & 1) * 2 + 1] = pack_pair<T>(p2, p3);
      }
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        s0 += __shfl_xor_sync(0xffffffffu, s0, off);
        s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      }
      l0 = fmaf(l0, a0, s0);
      l1 = fmaf(l1, a1, s1);
#pragma unroll
      for (int nt = 0; nt < NO; ++nt) {
        o[nt][0] *= a0;
        o[nt][1] *= a0;
        o[nt][2] *= a1;
        o[nt][3] *= a1;
      }
      // ---- O += P V
      const int rV = rK + 1, sV = warp * NR + rV % NR;
      if (!wait(bar_full(sV), static_cast<uint32_t>(rV / NR) & 1u)) {
        ok = false;
        break;
      }
      const uint32_t vb = slot(sV);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
#pragma unroll
        for (int nt = 0; nt < NO; nt += 2) {
          uint32_t b[4];  // b0, b1 of column tile nt, then of nt + 1
          ldsm_x4_trans(vb + dt_off(ks * 16 + (mi & 1) * 8 + rr, (nt + (mi >> 1)) * 8), b);
          mma16816<T>(o[nt], pa[ks], b[0], b[1]);
          mma16816<T>(o[nt + 1], pa[ks], b[2], b[3]);
        }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty(sV));
    }
    if (!ok) break;
    // ---- the chunk's partial: O / l and the base-2 LSE, per valid query head
    const float inv0 = l0 > 0.f ? 1.0f / l0 : 0.f, inv1 = l1 > 0.f ? 1.0f / l1 : 0.f;
    const int64_t grow0 = static_cast<int64_t>(ch.b) * p.H + h0 + g;
#pragma unroll
    for (int nt = 0; nt < NO; ++nt) {
      const int d = nt * 8 + 2 * q;
      if (row0)
        *reinterpret_cast<float2*>(p.part_o + (grow0 * p.n_splits + ch.c) * D + d) =
            make_float2(o[nt][0] * inv0, o[nt][1] * inv0);
      if (row1)
        *reinterpret_cast<float2*>(p.part_o + ((grow0 + 8) * p.n_splits + ch.c) * D + d) =
            make_float2(o[nt][2] * inv1, o[nt][3] * inv1);
    }
    if (q == 0) {
      if (row0) p.part_lse[grow0 * p.n_splits + ch.c] = l0 > 0.f ? m0 + lg2_approx(l0) : -INFINITY;
      if (row1) p.part_lse[(grow0 + 8) * p.n_splits + ch.c] = l1 > 0.f ? m1 + lg2_approx(l1) : -INFINITY;
    }
  }
}

}  // namespace flexattn
