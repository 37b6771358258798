// flex_fwd_fp8_sm100.cuh -- flex-attention forward with 8-bit (e4m3) Q, K, V for sm_100a.
//
// FP8 flex paths are named as a later phase on FlyDSL PR 931 "Add flex_attention
// (score_mod / mask_mod) on the generic flash-attention kernel" (Out of scope).  Inputs are
// e4m3 codes with per-tensor descales (q = descale_q * q8, ...); O is bf16, LSE fp32:
//   O = softmax(mask_mod(score_mod(scale * q.k))) v,   computed as
//   S = q8 k8^T (tcgen05 kind::f8f6f4, fp32 in TMEM) * (scale * descale_q * descale_k),
//   P rounded to e4m3 for the P.V product, O = descale_v * (P v8) / l.
// The structure is the 16-bit kernel's (two 128-row query tiles per CTA, one MMA-issuing
// thread, a TMA producer that publishes step records, two softmax warpgroups, the same
// visit sets for block masks and document masks, the same debug tile map), with two
// differences that keep both operands of every product K-major, the form every tcgen05
// kind accepts:
//   - P goes through shared memory (each softmax thread writes its row's 128 e4m3 values
//     in the 128-byte-swizzled layout, then fences the async proxy) instead of TMEM;
//   - V is read as V^T tiles [128 dims x 128 keys] from a transposed copy that
//     fp8_transpose_v_kernel writes first (keys padded to a multiple of 128 with zeros).
// P is computed as 2^(x - m + 6) with the O rescale threshold at 2^2, so its largest value
// is 2^8 <= 448 (the e4m3 maximum) and values down to 2^-15 of the row maximum survive the
// 8-bit rounding; the factor 2^6 cancels between O and l.  Head dim 128 or 64: tiles are
// always 128 bytes wide; at D = 64 the TMA boxes of Q and K run past the 64-byte rows and
// the V^T box past its 64 rows, and TMA fills those bytes with zeros, so S gains only zero
// products and O's columns 64..127 stay zero (they are not stored).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include <cstdint>

#include "flex_fwd_sm100.cuh"
#include "mask_rules.cuh"
#include "ptx_sm100.cuh"

namespace flexattn {

constexpr int kFp8D = 128;  // width of every 8-bit tile in bytes (head dims 64 and 128 fit)
constexpr float kP8Shift = 6.0f;      // log2 of the factor P carries into the 8-bit product
constexpr float kP8Rescale = 2.0f;    // O rescale threshold (log2) for the 8-bit path
#ifndef FLEX_FP8_EMU_PAIRS
#define FLEX_FP8_EMU_PAIRS 0
#endif
// Of the 8 value pairs of each 16-key chunk, how many take 2^x from the polynomial on the
// FMA pipe instead of MUFU ex2 (the 8-bit kernel is bound by MUFU, not the tensor core).
constexpr int kFp8EmuPairs = FLEX_FP8_EMU_PAIRS;

struct Fp8Params {
  __nv_bfloat16* o;
  float* lse;
  uint8_t* tile_map;  // debug tile map or nullptr
  unsigned* status;
  int H, Hkv, G, Sq, Skv, Skv_pad, D;
  int n_qtiles, n_ktiles, n_pairs;
  int bh_total, head_group;  // B * H; units run in groups of head_group heads (unit_coords_of)
  float scale_log2;   // scale * descale_q * descale_k * log2(e)
  float descale_v;
  const float* slopes;
  MaskArgs mask;      // document rules: boundaries of batch 0, advanced per batch
  VisitLists blocks;  // block mask (BLOCKS instantiations)
};

template <bool BLOCKS = false, bool DOC = false>
struct Fp8Smem {
  static constexpr int kTileBytes = kBM * kFp8D;  // 128 rows x 128 bytes
  static constexpr int kSlots = 10;               // K / V^T ring
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kPOff = kKVOff + kSlots * kTileBytes;
  static constexpr int kBarOff = kPOff + 2 * kTileBytes;
  // barriers: q, full[NS], empty[NS], s_full[2], p_half[2][2], o_full[2], drain
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 4 + 2 + 1;
  static constexpr int kTmemPtrOff = kBarOff + kNumBars * 8;
  static constexpr int kRecOff = kTmemPtrOff + 16;
  static constexpr int kRecBytes = ((kSlots + 1) * 4 + 15) / 16 * 16;
  // document rules: the documents of each tile's first and last row; then the visit sets
  static constexpr int kDocOff = kRecOff + kRecBytes;
  static constexpr int kBlkOff = kDocOff + (DOC ? 16 : 0);
  static constexpr int kBytes = kBlkOff + fwd_bitmaps(BLOCKS, DOC) * kBlkWords * 4;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA exceeded");
};

// D[tmem] (+)= A[smem] * B[smem], 8-bit operands (kind::f8f6f4)
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Generic-proxy writes to shared memory become visible to the tensor core's reads.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

// V [rows, Skv, D] bytes -> V^T [rows, D, Skv_pad] bytes (keys past Skv are zero).
// One CTA per (row, 128-key tile), 256 threads.  (A template so that every translation
// unit that sees this header shares one definition.)
template <int D>
__global__ void __launch_bounds__(256) fp8_transpose_v_kernel(const uint8_t* v, uint8_t* vt, int Skv, int Skv_pad,
                                                              int n_tiles) {
  static_assert(D == 64 || D == 128, "the 8-bit path has head dim 64 or 128");
  constexpr int kPieces = D / 16;  // 16-byte pieces of one key row
  __shared__ uint8_t tile[128][D + 16];
  const int64_t row = blockIdx.x / n_tiles;
  const int j0 = (blockIdx.x % n_tiles) * 128;
  const uint8_t* src = v + row * static_cast<int64_t>(Skv) * D;
  for (int e = threadIdx.x; e < 128 * kPieces; e += 256) {  // 16-byte pieces of 128 key rows
    const int jj = e / kPieces, piece = e % kPieces;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (j0 + jj < Skv) val = *reinterpret_cast<const uint4*>(src + static_cast<int64_t>(j0 + jj) * D + piece * 16);
    const uint8_t* b = reinterpret_cast<const uint8_t*>(&val);
#pragma unroll
    for (int x = 0; x < 16; ++x) tile[jj][piece * 16 + x] = b[x];
  }
  __syncthreads();
  uint8_t* dst = vt + row * static_cast<int64_t>(D) * Skv_pad;
  for (int e = threadIdx.x; e < D * 8; e += 256) {  // dim d, 16 consecutive keys
    const int d = e >> 3, piece = e & 7;
    alignas(16) uint8_t b[16];
#pragma unroll
    for (int x = 0; x < 16; ++x) b[x] = tile[piece * 16 + x][d];
    *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(d) * Skv_pad + j0 + piece * 16) =
        *reinterpret_cast<const uint4*>(b);
  }
}

template <int SCORE, int MASK, bool BLOCKS>
__global__ void __launch_bounds__(kFwdThreads, 1)
    flex_fwd_fp8_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmVt, const Fp8Params p) {
  constexpr bool kDoc = is_doc_mask(MASK);
  constexpr bool kBits = BLOCKS || kDoc;
  using L = Fp8Smem<BLOCKS, kDoc>;
  constexpr int NS = L::kSlots;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kIdesc = idesc_f16(0, kBM, kBN, 0);  // e4m3 x e4m3 -> f32, both K-major

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_addr);
  const uint32_t bar_q = sbase + L::kBarOff;
  auto bar_full = [&](int s) { return sbase + L::kBarOff + 8u * (1 + s); };
  auto bar_empty = [&](int s) { return sbase + L::kBarOff + 8u * (1 + NS + s); };
  auto bar_s = [&](int k) { return sbase + L::kBarOff + 8u * (1 + 2 * NS + k); };
  auto bar_p = [&](int k, int half) { return sbase + L::kBarOff + 8u * (3 + 2 * NS + 2 * k + half); };
  auto bar_o = [&](int k) { return sbase + L::kBarOff + 8u * (7 + 2 * NS + k); };
  const uint32_t bar_drain = sbase + L::kBarOff + 8u * (9 + 2 * NS);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sgen + L::kTmemPtrOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kTmemPtrOff + 4);
  uint32_t* rec_smem = reinterpret_cast<uint32_t*>(sgen + L::kRecOff);
  auto q_smem = [&](int k) { return sbase + static_cast<uint32_t>(L::kQOff + k * L::kTileBytes); };
  auto kv_smem = [&](int s) { return sbase + static_cast<uint32_t>(L::kKVOff + s * L::kTileBytes); };
  auto p_smem = [&](int k) { return sbase + static_cast<uint32_t>(L::kPOff + k * L::kTileBytes); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bh, pair;
  unit_coords_of(static_cast<int>(blockIdx.x), p.n_pairs, p.head_group, p.bh_total, bh, pair);
  const int h = bh % p.H, b = bh / p.H;
  const int bkv = b * p.Hkv + h / p.G;
  int q0[2], q1[2], lo[2], hi[2];
  auto sel = [](const int (&a)[2], int k) { return k ? a[1] : a[0]; };
  MaskArgs mk = p.mask;
  if constexpr (kDoc) {
    mk.off_q += static_cast<int64_t>(b) * (mk.n_docs + 1);
    mk.off_kv += static_cast<int64_t>(b) * (mk.n_docs + 1);
  }
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const int qt = 2 * pair + k;
    q0[k] = qt * kBM;
    q1[k] = min(q0[k] + kBM, p.Sq);
    lo[k] = hi[k] = 0;
    if (qt < p.n_qtiles && !kDoc) tile_range<MASK>(q0[k], q1[k], kBN, mk, lo[k], hi[k]);
  }
  // visit sets of the two query tiles (block masks, document masks), as in the 16-bit kernel
  uint32_t* blk = reinterpret_cast<uint32_t*>(sgen + L::kBlkOff);
  if constexpr (kBits)
    build_visit_sets<MASK, BLOCKS>(blk, reinterpret_cast<int*>(sgen + L::kDocOff), p.blocks, pair, b, h, q0, q1, lo,
                                   hi, mk, p.n_qtiles, p.n_ktiles, p.Skv);
  auto cursor = [&](int k) {
    if constexpr (kBits) return BitCursor(visit_act_bits(blk, k), visit_full_bits(blk, k), p.n_ktiles);
    else return RangeCursor(sel(lo, k), sel(hi, k));
  };
  auto has = [&](int k, int j) -> bool {  // debug tile map only
    if constexpr (kBits) return bits_has(visit_act_bits(blk, k), j);
    else return j >= sel(lo, k) && j < sel(hi, k);
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar_s(k), 1);
      mbar_init(bar_p(k, 0), kBM);
      mbar_init(bar_p(k, 1), kBM);
      mbar_init(bar_o(k), 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_ptr), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const bool act0 = cursor(0).cur >= 0, act1 = cursor(1).cur >= 0;
  const bool any_work = act0 || act1;

  if (warp < kSoftmaxWarp0) {
    regs_dec<kAuxRegs>();
    if (warp == kTmaWarp && lane == 0 && any_work) {
      // ============================================================ TMA producer
      int r = 0;
      bool ok = true;
      auto c0 = cursor(0), c1 = cursor(1);
      auto make_rec = [](auto a0, auto a1) -> uint32_t {
        const int j = max(a0.cur, a1.cur);
        if (j < 0) return kRecEnd;
        const bool i0 = a0.cur == j, i1 = a1.cur == j;
        if (i0) a0.advance();
        if (i1) a1.advance();
        const int jn = max(a0.cur, a1.cur);
        uint32_t rec = (i0 ? kRecIn0 : 0u) | (i1 ? kRecIn1 : 0u);
        if (i0) rec |= a0.cur < 0 ? kRecLast0 : (a0.cur == jn ? kRecPre0 : 0u);
        if (i1) rec |= a1.cur < 0 ? kRecLast1 : (a1.cur == jn ? kRecPre1 : 0u);
        return rec;
      };
      rec_smem[NS] = make_rec(c0, c1);
      mbar_arrive_expect_tx(bar_q, (act0 ? L::kTileBytes : 0) + (act1 ? L::kTileBytes : 0));
      if (act0) tma_load_3d(q_smem(0), &tmQ, bar_q, 0, q0[0], bh);
      if (act1) tma_load_3d(q_smem(1), &tmQ, bar_q, 0, q0[1], bh);
      for (int j = max(c0.cur, c1.cur); j >= 0 && ok; j = max(c0.cur, c1.cur)) {
        if (c0.cur == j) c0.advance();
        if (c1.cur == j) c1.advance();
        const uint32_t next_rec = make_rec(c0, c1);
        for (int which = 0; which < 2 && ok; ++which, ++r) {
          const int s = r % NS;
          if (!mbar_wait(bar_empty(s), (static_cast<uint32_t>(r / NS) & 1u) ^ 1u, p.status, kStatusFwdTimeout,
                         kWaitTimeoutNs) ||
              *abort_flag) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          if (which == 1) rec_smem[s] = next_rec;
          mbar_arrive_expect_tx(bar_full(s), L::kTileBytes);
          if (which == 0)
            tma_load_3d(kv_smem(s), &tmK, bar_full(s), 0, j * kBN, bkv);       // K [128 keys x 128 dims]
          else
            tma_load_3d(kv_smem(s), &tmVt, bar_full(s), j * kBN, 0, bkv);      // V^T [128 dims x 128 keys]
        }
      }
      for (int e = r - NS < 0 ? 0 : r - NS; e < r; ++e)
        mbar_wait(bar_full(e % NS), static_cast<uint32_t>(e / NS) & 1u, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
      mbar_wait(bar_q, 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
    } else if (warp == kMmaWarp && lane == 0 && any_work) {
      // ============================================================ MMA issuer
      bool ok = mbar_wait(bar_q, 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
      tc_fence_after();
      int np[2] = {0, 0};
      // 32 e4m3 values (32 bytes) per k-step inside one 128-byte swizzled row
      auto issue_s = [&](int k, int slot) {
        const uint64_t aq = smem_desc(q_smem(k), 16, 1024, kSwizzle128B);
        const uint64_t bk = smem_desc(kv_smem(slot), 16, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = 0; kk < kFp8D / 32; ++kk)
          mma_ss_f8(tmem + 128u * k, aq + static_cast<uint64_t>(kk * 2), bk + static_cast<uint64_t>(kk * 2), kIdesc,
                    kk > 0 ? 1u : 0u);
      };
      auto issue_pv = [&](int k, int slot, bool acc, int kk0, int kk1) {
        const uint64_t ap = smem_desc(p_smem(k), 16, 1024, kSwizzle128B);
        const uint64_t bv = smem_desc(kv_smem(slot), 16, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk)
          mma_ss_f8(tmem + 256u + 128u * k, ap + static_cast<uint64_t>(kk * 2), bv + static_cast<uint64_t>(kk * 2),
                    kIdesc, (acc || kk > 0) ? 1u : 0u);
      };
      bool s_ready[2] = {false, false}, started[2] = {false, false};
      auto tile_step = [&](auto kc, bool pre, bool last, int rK, int sV, bool& next_k_ready) -> bool {
        constexpr int k = decltype(kc)::value;
        s_ready[k] = false;
        const uint32_t par = static_cast<uint32_t>(np[k]) & 1u;
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(bar_p(k, half), par, p.status, kStatusFwdTimeout, kWaitTimeoutNs)) return false;
          tc_fence_after();
          issue_pv(k, sV, started[k], 2 * half, 2 * half + 2);
        }
        started[k] = true;
        ++np[k];
        if (pre) {
          const int rK2 = rK + 2;
          if (!next_k_ready) {
            if (!mbar_wait(bar_full(rK2 % NS), static_cast<uint32_t>(rK2 / NS) & 1u, p.status, kStatusFwdTimeout,
                           kWaitTimeoutNs))
              return false;
            tc_fence_after();
            next_k_ready = true;
          }
          issue_s(k, rK2 % NS);
          mma_commit(bar_s(k));
          s_ready[k] = true;
        } else if (last) {
          mma_commit(bar_o(k));
        }
        return true;
      };
      uint32_t rec = rec_smem[NS];
      for (int t = 0; !(rec & kRecEnd) && ok; ++t) {
        const int rK = 2 * t, rV = rK + 1;
        const int sK = rK % NS, sV = rV % NS;
        const bool in0 = rec & kRecIn0, in1 = rec & kRecIn1;
        const bool need0 = in0 && !s_ready[0], need1 = in1 && !s_ready[1];
        if (need0 || need1) {
          if (!mbar_wait(bar_full(sK), static_cast<uint32_t>(rK / NS) & 1u, p.status, kStatusFwdTimeout,
                         kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (need0) {
            issue_s(0, sK);
            mma_commit(bar_s(0));
          }
          if (need1) {
            issue_s(1, sK);
            mma_commit(bar_s(1));
          }
        }
        mma_commit(bar_empty(sK));
        if (!mbar_wait(bar_full(sV), static_cast<uint32_t>(rV / NS) & 1u, p.status, kStatusFwdTimeout,
                       kWaitTimeoutNs)) {
          ok = false;
          break;
        }
        const uint32_t next_rec = rec_smem[sV];
        bool next_k_ready = false;
        if (in0)
          ok = tile_step(std::integral_constant<int, 0>{}, rec & kRecPre0, rec & kRecLast0, rK, sV, next_k_ready);
        if (ok && in1)
          ok = tile_step(std::integral_constant<int, 1>{}, rec & kRecPre1, rec & kRecLast1, rK, sV, next_k_ready);
        if (!ok) break;
        mma_commit(bar_empty(sV));
        rec = next_rec;
      }
      if (!ok) *abort_flag = 1;
      mma_commit(bar_drain);
      mbar_wait(bar_drain, 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
    }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ============================================================ softmax warpgroups
    const int k = (warp - kSoftmaxWarp0) >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int q0k = sel(q0, k), q1k = sel(q1, k);
    const int qi = q0k + row;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128u * k;
    const uint32_t tO = tmem + lane_off + 256u + 128u * k;
    const bool tile_valid = (2 * pair + k) < p.n_qtiles;
    const bool act_k = k == 0 ? act0 : act1;
    const int qt = 2 * pair + k;
    const bool write_map = p.tile_map != nullptr && bh == 0 && tile_valid && threadIdx.x % 128 == 0;
    if (write_map) {
      for (int u = 0; u < p.n_ktiles; ++u)
        if (!act_k || !has(k, u)) p.tile_map[static_cast<int64_t>(qt) * p.n_ktiles + u] = kTileEmpty;
    }
    // Document rules: this row's kept interval, looked up once.
    int64_t row_lo = 0, row_hi = -1;
    if constexpr (kDoc) row_interval<MASK>(qi, mk, row_lo, row_hi);
    // this thread's row of P in the 128-byte-swizzled tile: chunk c lives at chunk c ^ (row % 8)
    uint8_t* prow = sgen + L::kPOff + k * L::kTileBytes + row * 128;
    const int swz = row & 7;

    float m_used = -INFINITY, l_sum = 0.f;
    const float sc = SCORE == kScoreAlibi ? 1.0f : p.scale_log2;
    float slope2 = 0.f;
    if (SCORE == kScoreAlibi)
      slope2 = (p.slopes ? __ldg(p.slopes + h) : exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(p.H))) *
               kLog2e;
    bool ok = true;
    int n = 0;
    auto cur = cursor(k);
    for (int j = act_k ? cur.cur : -1; j >= 0; j = cur.cur, ++n) {
      // with block masks and document masks the class comes from the walk
      const int cls_blk = cur.cur_full ? (j * kBN + kBN > p.Skv ? kTileFullRagged : kTileFull) : kTilePartial;
      cur.advance();
      const bool got = mbar_wait(bar_s(k), static_cast<uint32_t>(n) & 1u, p.status, kStatusFwdTimeout,
                                 kWaitTimeoutNs) &&
                       !*abort_flag;
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = j * kBN;
      int cls;
      if constexpr (kBits) cls = cls_blk;
      else cls = tile_class<MASK>(q0k, q1k, k0, kBN, mk);
      if (write_map)
        p.tile_map[static_cast<int64_t>(qt) * p.n_ktiles + j] =
            static_cast<uint8_t>(cls == kTileFullRagged ? kTilePartial : cls);
      uint32_t sr[kBN];
      tmem_ld128(tS, sr);
      float* s = reinterpret_cast<float*>(sr);
      if (SCORE == kScoreAlibi) {  // scale folded here; otherwise into the exponent below
        const float base = slope2 * static_cast<float>(k0 - qi);
#pragma unroll
        for (int c = 0; c < kBN; ++c) s[c] = fmaf(s[c], p.scale_log2, fmaf(slope2, static_cast<float>(c), base));
      }
      if (cls != kTileFull) {
        int c_lo, c_hi;
        if (kBits && cls == kTileFullRagged)
          col_interval<kMaskNone>(qi, k0, mk, c_lo, c_hi);
        else if constexpr (kDoc)
          col_interval_of(row_lo, row_hi, k0, c_lo, c_hi);
        else
          col_interval<MASK>(qi, k0, mk, c_lo, c_hi);
#pragma unroll
        for (int c = 0; c < kBN; ++c)
          if (c < c_lo || c > c_hi) s[c] = -INFINITY;
      }
      float mx0 = max3f(s[0], s[1], s[2]), mx1 = max3f(s[3], s[4], s[5]);
      float mx2 = max3f(s[6], s[7], s[8]), mx3 = max3f(s[9], s[10], s[11]);
#pragma unroll
      for (int c = 12; c + 8 <= kBN - 4; c += 8) {
        mx0 = max3f(mx0, s[c], s[c + 1]);
        mx1 = max3f(mx1, s[c + 2], s[c + 3]);
        mx2 = max3f(mx2, s[c + 4], s[c + 5]);
        mx3 = max3f(mx3, s[c + 6], s[c + 7]);
      }
      mx0 = max3f(mx0, s[kBN - 4], s[kBN - 3]);
      mx1 = max3f(mx1, s[kBN - 2], s[kBN - 1]);
      const float mx = max3f(mx0, mx1, fmaxf(mx2, mx3)) * sc;
      const bool need = mx > m_used + kP8Rescale;
      if (__any_sync(0xffffffffu, need)) {
        float alpha = 1.0f;
        if (need) {
          alpha = ex2_approx(m_used - mx);
          m_used = mx;
          l_sum *= alpha;
        }
        if (n > 0) {
          const uint64_t a2 = pack2(alpha, alpha);
#pragma unroll 1
          for (int c = 0; c < kFp8D; c += 32) {
            uint32_t r[32];
            tmem_ld32(tO + c, r);
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const uint64_t v = mul2(pack2(__uint_as_float(r[e]), __uint_as_float(r[e + 1])), a2);
              r[e] = static_cast<uint32_t>(v);
              r[e + 1] = static_cast<uint32_t>(v >> 32);
            }
            tmem_st32(tO + c, r);
          }
        }
      }
      // 2^(s * sc - m + 6): P carries 2^6 into the 8-bit product (cancels against l)
      const float nm = kP8Shift - (m_used == -INFINITY ? 0.f : m_used);
      const uint64_t sc2 = pack2(sc, sc), nm2 = pack2(nm, nm);
      uint64_t acc_a = 0, acc_b = 0;  // four running partial sums of P
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {  // 16 keys per 16-byte chunk
          const int c0 = 64 * half + 16 * ch;
          float e[16];
#pragma unroll
          for (int x = 0; x < 16; x += 2) {
            const uint64_t x2 = fma2(pack2(s[c0 + x], s[c0 + x + 1]), sc2, nm2);
            if (x / 2 >= 8 - kFp8EmuPairs) {  // this pair on the FMA pipe
              unpack2(exp2_poly2(x2), e[x], e[x + 1]);
            } else {
              float x0, x1;
              unpack2(x2, x0, x1);
              e[x] = ex2_approx(x0);
              e[x + 1] = ex2_approx(x1);
            }
            if (x & 2)
              acc_b = add2(acc_b, pack2(e[x], e[x + 1]));
            else
              acc_a = add2(acc_a, pack2(e[x], e[x + 1]));
          }
          const uint4 w = make_uint4(e4m3x4(e[0], e[1], e[2], e[3]), e4m3x4(e[4], e[5], e[6], e[7]),
                                     e4m3x4(e[8], e[9], e[10], e[11]), e4m3x4(e[12], e[13], e[14], e[15]));
          *reinterpret_cast<uint4*>(prow + (((4 * half + ch) ^ swz) << 4)) = w;
        }
        fence_proxy_async_smem();
        mbar_arrive(bar_p(k, half));
      }
      float a0, a1, b0, b1;
      unpack2(acc_a, a0, a1);
      unpack2(acc_b, b0, b1);
      l_sum += (a0 + a1) + (b0 + b1);
    }
    if (!ok) *abort_flag = 1;

    if (tile_valid) {
      bool ran = ok && act_k;
      if (ran) {
        const bool got = mbar_wait(bar_o(k), 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
        if (!__all_sync(0xffffffffu, got)) {
          *abort_flag = 1;
          ran = false;
        }
        tc_fence_after();
      }
      const bool row_ok = qi < p.Sq;
      const bool has_mass = ran && m_used != -INFINITY && l_sum > 0.f;
      const float inv = has_mass ? p.descale_v / l_sum : 0.f;
      __nv_bfloat16* orow = p.o + (static_cast<int64_t>(bh) * p.Sq + qi) * p.D;
#pragma unroll 1
      for (int c = 0; c < p.D; c += 32) {
        uint32_t r[32];
        if (ran) tmem_ld32(tO + c, r);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = DtypeBits<__nv_bfloat16>::pack(has_mass ? __uint_as_float(r[2 * e]) * inv : 0.f,
                                                has_mass ? __uint_as_float(r[2 * e + 1]) * inv : 0.f);
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
      if (row_ok && p.lse != nullptr)
        p.lse[static_cast<int64_t>(bh) * p.Sq + qi] =
            has_mass ? (m_used - kP8Shift + lg2_approx(l_sum)) * kLn2 : -INFINITY;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace flexattn
