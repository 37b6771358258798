// flex_bwd_sm100.cuh -- flex-attention backward for sm_100a: dQ, dK, dV of sum(dO * O).
//
// The backward pass is named as a later phase on FlyDSL PR 931 "Add flex_attention
// (score_mod / mask_mod) on the generic flash-attention kernel" (Out of scope); xformers
// 1094 "Tiny upstream pr" reports dq/dk/dv errors of a backward against a reference.
// With the forward's LSE (natural log) and O, per query row i and kept key j:
//   P_ij = exp(x_ij - LSE_i),  delta_i = dO_i . O_i,  dP_ij = dO_i . V_j,
//   dS_ij = P_ij (dP_ij - delta_i),
//   dQ_i = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,  dV_j = sum_i P_ij dO_i
// (dK, dV summed over the query heads of a GQA group); x_ij is the forward's modded,
// scaled score, so the mods enter through P and the masks zero P.
//
// Three kernels, no atomics (results do not depend on scheduling):
//   bwd_prep_kernel   per row: -delta_i and -LSE_i * log2(e) into a padded workspace
//   bwd_dq_kernel     one CTA per 128-row query tile: for each key tile, S = Q K^T and
//                     dP = dO V^T (tcgen05, TMEM), dS on the CUDA cores (one row per
//                     thread), dQ += dS K (tcgen05, dS read from TMEM); S alternates between
//                     two TMEM buffers so S of the next key tile overlaps the dS work, and
//                     K and V stream through rings of their own, each freed in order
//   bwd_dkdv_kernel   one CTA per 128-key tile and kv head: for each query tile of each
//                     query head of the group, S^T = K Q^T and dP^T = V dO^T, P^T and dS^T
//                     per key row, dV += P^T dO and dK += dS^T Q (TMEM accumulators)
// With a block mask (BLOCKS instantiations; BlockMask, named with the backward as later
// phases on FlyDSL PR 931, Out of scope) the keep rule is the block-sparse forward's: a
// key tile on a query tile's full list keeps every key below Skv, one on its partial list
// the keys mask_mod keeps.  The dQ kernel walks its query tile's listed key tiles from
// bitmaps it builds in shared memory; the dK/dV kernel walks the (query head, query tile)
// pairs that list its key tile, from transposed bitmaps that bwd_block_transpose_kernel
// writes into the workspace first (one atomicOr per listed block, so the transpose costs
// the size of the lists, not a scan per key tile).
// Roles per CTA (384 threads): warp 0 issues the MMAs (one thread), warp 1 the TMA loads,
// warps 4-7 and 8-11 do the element-wise work on the two 64-column halves of each tile
// (thread = TMEM lane = row), warps 2-3 idle.  Each half writes its 16-bit results into
// its own quarter of the TMEM buffer it read (columns [0, 32) and [64, 96)), and signals
// its own barrier, so the products that consume them start on the first finished half.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "flex_fwd_sm100.cuh"
#include "mask_rules.cuh"
#include "ptx_sm100.cuh"

namespace flexattn {

constexpr int kBwdThreads = 384;
constexpr int kBwdWarp0 = 4;  // warps 4-7: columns [0, 64) of each tile, warps 8-11: [64, 128)
constexpr unsigned kStatusBwdTimeout = 16u;

struct BwdParams {
  const void* o;          // forward output [B, H, Sq, D]
  const void* dout;       // upstream gradient [B, H, Sq, D]
  const float* lse;       // forward LSE [B, H, Sq] (natural log)
  float* nlse2;           // workspace [B*H, Sq_pad]: -LSE * log2(e), -inf for rows without keys
  float* ndelta;          // workspace [B*H, Sq_pad]: -(dO . O)
  void* dq;               // [B, H, Sq, D]
  void* dk;               // [B, Hkv, Skv, D]
  void* dv;               // [B, Hkv, Skv, D]
  unsigned* status;
  int B, H, Hkv, G, Sq, Skv, D, Sq_pad;
  int n_qtiles, n_ktiles;
  // CTA order (unit_coords_of): the dQ kernel runs head by head with its query tiles in
  // order (q_group 0), or under causal-like masks the last (heaviest) query tiles first
  // over groups of q_group query heads; the dK/dV kernel runs its key tiles in order over
  // groups of kv_group kv heads (1: head by head; under causal masks the first key tiles
  // see the most queries)
  int q_group, kv_group;
  float scale;
  float scale_log2;       // scale * log2(e)
  const float* slopes;    // alibi slope tensor [H] or nullptr
  MaskArgs mask;          // document rules: boundaries of batch 0, advanced per batch
  // Block mask (BLOCKS instantiations), as in FwdParams: [0] partial, [1] full lists.
  const int32_t* blk_num[2];
  const int32_t* blk_idx[2];
  int blk_max, blk_b_stride, blk_h_stride;
  // Transposed block mask in the workspace: per (b, kv head, key tile) two bitmaps of
  // tb_words words over the (query head in group, query tile) pairs hg * n_qtiles + t:
  // tbits[row * 2 * tb_words + w] (pairs that visit the key tile) and
  // tbits[row * 2 * tb_words + tb_words + w] (those whose visit is FULL).
  uint32_t* tbits;
  int tb_words;
};

// Block-mask bitmap words a dQ CTA keeps in shared memory (key tiles <= 32 * kBwdBlkWords).
constexpr int kBwdBlkWords = kBlkWords;

// Ascending walk over the set bits of a bitmap (words read through `load`), with the
// companion bitmap's bit of each position in cur_full; cur = -1 once the walk is over.
template <typename Load>
struct AscBits {
  Load load;
  int n_words, wi;
  uint32_t bits, cword;
  int cur;
  bool cur_full;
  __device__ __forceinline__ AscBits(Load l, int nw) : load(l), n_words(nw), wi(-1), bits(0), cword(0), cur(-1),
                                                        cur_full(false) {
    advance();
  }
  __device__ __forceinline__ void advance() {
    while (bits == 0) {
      if (++wi >= n_words) {
        cur = -1;
        return;
      }
      bits = load(wi, 0);
      cword = load(wi, 1);
    }
    const int bit = __ffs(bits) - 1;
    bits &= bits - 1u;
    cur = (wi << 5) + bit;
    cur_full = (cword >> bit) & 1u;
  }
};
template <typename Load>
__device__ __forceinline__ AscBits<Load> asc_bits(Load l, int n_words) {
  return AscBits<Load>(l, n_words);
}

// The class a block mask gives key tile u of query tile [q0, q1): -1 (the tile keeps
// nothing), kTileFull (every key below Skv kept) or kTilePartial (mask_mod per element).
// A block on the full list is FULL; a partial block that mask_mod drops whole keeps
// nothing and one it keeps whole is FULL, as in the forward (document rules: partial).
template <int MASK>
__device__ __forceinline__ int block_tile_class(bool listed_full, int q0, int q1, int u, const MaskArgs& m) {
  if (listed_full) return kTileFull;
  if constexpr (MASK == kMaskDocument || MASK == kMaskDocumentCausal) {
    return kTilePartial;
  } else {
    int lo, hi;
    tile_range<MASK>(q0, q1, kBN, m, lo, hi);
    if (u < lo || u >= hi) return -1;
    return tile_class<MASK>(q0, q1, u * kBN, kBN, m) == kTileFull ? kTileFull : kTilePartial;
  }
}

// ---------------------------------------------------------------- block-mask transpose

// One warp per list row (b, h, t): every key tile u the row lists sets bit hg * n_qtiles
// + t of the (b, kv head, u) bitmaps in the workspace (zeroed before the launch), and of
// the FULL bitmap when the visit needs no element mask.  Counts are clamped and indices
// range-checked as in the forward.
template <int MASK>
__global__ void __launch_bounds__(256) bwd_block_transpose_kernel(const BwdParams p) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.n_qtiles;
  const int lane = threadIdx.x & 31;
  for (int64_t r = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; r < rows;
       r += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int t = static_cast<int>(r % p.n_qtiles);
    const int64_t bh = r / p.n_qtiles;
    const int h = static_cast<int>(bh % p.H), b = static_cast<int>(bh / p.H);
    const int hk = h / p.G, hg = h % p.G;
    const int q0 = t * kBM, q1 = min(q0 + kBM, p.Sq);
    MaskArgs mk = p.mask;
    if constexpr (MASK == kMaskDocument || MASK == kMaskDocumentCausal) {
      mk.off_q += static_cast<int64_t>(b) * (mk.n_docs + 1);
      mk.off_kv += static_cast<int64_t>(b) * (mk.n_docs + 1);
    }
    const int64_t lrow = (static_cast<int64_t>(b) * p.blk_b_stride + static_cast<int64_t>(h) * p.blk_h_stride) *
                             p.n_qtiles + t;
    const int pair = hg * p.n_qtiles + t;
    for (int f = 0; f < 2; ++f) {
      const int32_t* num = f ? p.blk_num[1] : p.blk_num[0];
      const int32_t* idx = f ? p.blk_idx[1] : p.blk_idx[0];
      if (num == nullptr) continue;
      int cnt = num[lrow];
      cnt = cnt < 0 ? 0 : (cnt > p.blk_max ? p.blk_max : cnt);
      for (int c = lane; c < cnt; c += 32) {
        const int u = idx[lrow * p.blk_max + c];
        if (u < 0 || u >= p.n_ktiles) continue;
        const int cls = block_tile_class<MASK>(f == 1, q0, q1, u, mk);
        if (cls < 0) continue;
        uint32_t* row = p.tbits + ((static_cast<int64_t>(b) * p.Hkv + hk) * p.n_ktiles + u) * 2 * p.tb_words;
        atomicOr(row + (pair >> 5), 1u << (pair & 31));
        if (cls == kTileFull) atomicOr(row + p.tb_words + (pair >> 5), 1u << (pair & 31));
      }
    }
  }
}

// ---------------------------------------------------------------- prep

// One warp per row (b, h, i) of the padded row space: delta = dO . O in fp32, and the
// base-2 LSE, both stored negated so that the element-wise passes add them with packed
// f32x2 arithmetic; padding rows get -inf and 0 so that they contribute nothing.
template <int D, typename T>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const BwdParams p) {
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.Sq_pad;
  const int lane = threadIdx.x & 31;
  for (int64_t r = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5; r < rows;
       r += (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5) {
    const int64_t bh = r / p.Sq_pad;
    const int i = static_cast<int>(r - bh * p.Sq_pad);
    float acc = 0.f, nl2 = -INFINITY;
    if (i < p.Sq) {
      const int64_t base = (bh * p.Sq + i) * D;
      const T* o = reinterpret_cast<const T*>(p.o) + base;
      const T* g = reinterpret_cast<const T*>(p.dout) + base;
      for (int d = lane; d < D; d += 32) acc = fmaf(static_cast<float>(o[d]), static_cast<float>(g[d]), acc);
      const float l = p.lse[bh * p.Sq + i];
      nl2 = l == -INFINITY ? -INFINITY : -l * kLog2e;
    }
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
    if (lane == 0) {
      p.ndelta[r] = i < p.Sq ? -acc : 0.f;
      p.nlse2[r] = nl2;
    }
  }
}

// ---------------------------------------------------------------- shared memory

template <int D, bool BLOCKS = false>
struct BwdDqSmem {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kChunkBytes = kBM * 128;
  // Separate K and V rings: K_t is read from S(t) (two tiles ahead) to dQ(t), V_t only by
  // dP(t), so each ring frees its slots in order and every load has an iteration of lead.
  static constexpr int kKSlots = D == 128 ? 3 : 6;
  static constexpr int kVSlots = D == 128 ? 2 : 4;
  static constexpr int kQOff = 0;                   // Q, then dO
  static constexpr int kKVOff = 2 * kTileBytes;     // K slots, then V slots
  static constexpr int kBarOff = kKVOff + (kKSlots + kVSlots) * kTileBytes;
  // barriers: q, full_k[KS], empty_k[KS], full_v[VS], empty_v[VS], sdp[2], ds[2], done
  static constexpr int kNumBars = 1 + 2 * (kKSlots + kVSlots) + 5;
  static constexpr int kTmemPtrOff = kBarOff + kNumBars * 8;
  // block mask: the visit and FULL bitmaps of this query tile's key tiles
  static constexpr int kBlkOff = kTmemPtrOff + 16;
  static constexpr int kBytes = kBlkOff + (BLOCKS ? 2 * kBwdBlkWords * 4 : 0);
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA exceeded");
};

template <int D>
struct BwdDkvSmem {
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kChunkBytes = kBM * 128;
  static constexpr int kStatBytes = 2 * kBM * 4;                      // -lse2[128], -delta[128]
  static constexpr int kSlotBytes = 2 * kTileBytes + kStatBytes;      // Q, dO, stats
  static constexpr int kSlots = D == 128 ? 2 : 4;
  static constexpr int kKOff = 0;                                     // K, then V
  static constexpr int kSlotOff = 2 * kTileBytes;
  static constexpr int kBarOff = kSlotOff + kSlots * kSlotBytes;
  // barriers: kv, full[NS], empty[NS], sdp[2], pds[2], done
  static constexpr int kNumBars = 1 + 2 * kSlots + 5;
  static constexpr int kTmemPtrOff = kBarOff + kNumBars * 8;
  static constexpr int kBytes = kTmemPtrOff + 16;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA exceeded");
  static_assert(kSlotBytes % 1024 == 0, "slots must keep the 1024-byte swizzle alignment");
};

// Bounded wait that also gives up when another role of the CTA has given up.  The fast
// path is a single probe of the barrier: on the MMA-issuing thread every shared-memory
// access between two matmuls idles the tensor pipe for about 100 cycles, so the abort flag
// is read only when the phase is not complete yet.
__device__ __forceinline__ bool bwd_wait(uint32_t bar, uint32_t parity, const BwdParams& p, volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  if (!mbar_wait(bar, parity, p.status, kStatusBwdTimeout, kWaitTimeoutNs)) {
    *abort_flag = 1;
    return false;
  }
  return true;
}

// ---------------------------------------------------------------- dQ

template <int D, typename T, int SCORE, int MASK, bool BLOCKS>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const BwdParams p) {
  using L = BwdDqSmem<D, BLOCKS>;
  constexpr int KS = L::kKSlots, VS = L::kVSlots;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kIdescS = idesc_f16(DtypeBits<T>::kFmt, kBM, kBN, 0);       // S: K-major B
  constexpr uint32_t kIdescHalf = idesc_f16(DtypeBits<T>::kFmt, kBM, kBN / 2, 0);  // dP halves
  constexpr uint32_t kIdescDq = idesc_f16(DtypeBits<T>::kFmt, kBM, D, 1);    // dQ: B = K, N-major
  constexpr bool kDoc = is_doc_mask(MASK);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_addr);
  const uint32_t bar_q = sbase + L::kBarOff;
  auto full_k = [&](int s) { return sbase + L::kBarOff + 8u * (1 + s); };
  auto empty_k = [&](int s) { return sbase + L::kBarOff + 8u * (1 + KS + s); };
  auto full_v = [&](int s) { return sbase + L::kBarOff + 8u * (1 + 2 * KS + s); };
  auto empty_v = [&](int s) { return sbase + L::kBarOff + 8u * (1 + 2 * KS + VS + s); };
  const uint32_t bar_sdp0 = sbase + L::kBarOff + 8u * (1 + 2 * KS + 2 * VS);
  auto bar_sdp = [&](int half) { return bar_sdp0 + 8u * half; };
  auto bar_ds = [&](int half) { return bar_sdp0 + 8u * (2 + half); };
  const uint32_t bar_done = bar_sdp0 + 32u;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sgen + L::kTmemPtrOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kTmemPtrOff + 4);
  const uint32_t q_smem = sbase + L::kQOff, o_smem = q_smem + L::kTileBytes;
  auto k_smem = [&](int s) { return sbase + static_cast<uint32_t>(L::kKVOff + s * L::kTileBytes); };
  auto v_smem = [&](int s) { return sbase + static_cast<uint32_t>(L::kKVOff + (KS + s) * L::kTileBytes); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int qt, bh;
  if (p.q_group > 0) {
    unit_coords_of(static_cast<int>(blockIdx.x), p.n_qtiles, p.q_group, p.B * p.H, bh, qt);
  } else {
    qt = blockIdx.x % p.n_qtiles;
    bh = blockIdx.x / p.n_qtiles;
  }
  const int h = bh % p.H, b = bh / p.H;
  const int bkv = b * p.Hkv + h / p.G;
  const int q0 = qt * kBM, q1 = min(q0 + kBM, p.Sq);
  MaskArgs mk = p.mask;
  if constexpr (kDoc) {
    mk.off_q += static_cast<int64_t>(b) * (mk.n_docs + 1);
    mk.off_kv += static_cast<int64_t>(b) * (mk.n_docs + 1);
  }
  int lo = 0, hi = 0;
  tile_range<MASK>(q0, q1, kBN, mk, lo, hi);
  // Block mask: the key tiles this query tile visits (act) and those it keeps whole
  // (full), as bitmaps built from its two lists; the walk is their set bits in ascending
  // order.  Otherwise: key tiles lo .. hi-1 in ascending order.
  uint32_t* act_bits = reinterpret_cast<uint32_t*>(sgen + L::kBlkOff);
  uint32_t* full_bits = act_bits + kBwdBlkWords;
  const int n_words = (p.n_ktiles + 31) >> 5;
  if constexpr (BLOCKS) {
    for (int w = threadIdx.x; w < 2 * kBwdBlkWords; w += kBwdThreads) act_bits[w] = 0u;
    __syncthreads();
    const int64_t lrow = (static_cast<int64_t>(b) * p.blk_b_stride + static_cast<int64_t>(h) * p.blk_h_stride) *
                             p.n_qtiles + qt;
    for (int e = threadIdx.x; e < 2 * p.blk_max; e += kBwdThreads) {
      const int f = e >= p.blk_max ? 1 : 0, c = e - f * p.blk_max;
      const int32_t* num = f ? p.blk_num[1] : p.blk_num[0];
      const int32_t* idx = f ? p.blk_idx[1] : p.blk_idx[0];
      if (num == nullptr) continue;
      const int cnt = num[lrow];
      if (c >= (cnt < 0 ? 0 : (cnt > p.blk_max ? p.blk_max : cnt))) continue;
      const int u = idx[lrow * p.blk_max + c];
      if (u < 0 || u >= p.n_ktiles) continue;
      const int cls = block_tile_class<MASK>(f == 1, q0, q1, u, mk);
      if (cls < 0) continue;
      atomicOr(act_bits + (u >> 5), 1u << (u & 31));
      if (cls == kTileFull) atomicOr(full_bits + (u >> 5), 1u << (u & 31));
    }
    __syncthreads();
    int cnt = 0;
    for (int w = 0; w < n_words; ++w) cnt += __popc(act_bits[w]);
    lo = 0;
    hi = cnt;
  }
  const int n = hi - lo;  // steps
  auto smem_words = [act_bits, full_bits](int w, int which) { return which ? full_bits[w] : act_bits[w]; };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < KS; ++s) {
      mbar_init(full_k(s), 1);
      mbar_init(empty_k(s), 1);
    }
    for (int s = 0; s < VS; ++s) {
      mbar_init(full_v(s), 1);
      mbar_init(empty_v(s), 1);
    }
    mbar_init(bar_sdp(0), 1);
    mbar_init(bar_sdp(1), 1);
    mbar_init(bar_ds(0), kBM);
    mbar_init(bar_ds(1), kBM);
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  // TMEM columns: S buffers [0,128) and [128,256), dP [256,384), dQ [384, 384+D)
  auto s_col = [](int t) { return 128u * static_cast<uint32_t>(t & 1); };
  constexpr uint32_t kDpCol = 256, kDqCol = 384;

  if (warp == 1 && lane == 0 && n > 0) {
    // ============================================================ TMA producer
    mbar_arrive_expect_tx(bar_q, 2 * L::kTileBytes);
    for (int c = 0; c < kChunks; ++c) {
      tma_load_3d(q_smem + c * L::kChunkBytes, &tmQ, bar_q, c * 64, q0, bh);
      tma_load_3d(o_smem + c * L::kChunkBytes, &tmO, bar_q, c * 64, q0, bh);
    }
    // Loads in the order the products need them: K_0, V_0, K_1, then V_{t+1}, K_{t+2}.
    // Block mask: the key tile of each load comes from a walk of the visit bitmap (one
    // walk for the K loads, one for the V loads).
    int nk = 0, nv = 0;
    auto walk_k = asc_bits(smem_words, BLOCKS ? n_words : 0);
    auto walk_v = asc_bits(smem_words, BLOCKS ? n_words : 0);
    auto load = [&](bool is_v, int tile) -> bool {
      const int i = is_v ? nv : nk;
      const int slot = i % (is_v ? VS : KS);
      const uint32_t full = is_v ? full_v(slot) : full_k(slot);
      const uint32_t empty = is_v ? empty_v(slot) : empty_k(slot);
      if (!bwd_wait(empty, (static_cast<uint32_t>(i / (is_v ? VS : KS)) & 1u) ^ 1u, p, abort_flag)) return false;
      mbar_arrive_expect_tx(full, L::kTileBytes);
      const uint32_t dst = is_v ? v_smem(slot) : k_smem(slot);
      int key_tile = lo + tile;
      if constexpr (BLOCKS) {
        auto& w = is_v ? walk_v : walk_k;
        key_tile = w.cur;
        w.advance();
      }
      for (int c = 0; c < kChunks; ++c)
        tma_load_3d(dst + c * L::kChunkBytes, is_v ? &tmV : &tmK, full, c * 64, key_tile * kBN, bkv);
      if (is_v) ++nv;
      else ++nk;
      return true;
    };
    bool ok = load(false, 0) && load(true, 0) && (n < 2 || load(false, 1));
    for (int t = 0; t + 1 < n && ok; ++t) ok = load(true, t + 1) && (t + 2 >= n || load(false, t + 2));
    // wait for the copies still in flight before the CTA may exit
    for (int e = nk - KS < 0 ? 0 : nk - KS; e < nk; ++e)
      mbar_wait(full_k(e % KS), static_cast<uint32_t>(e / KS) & 1u, p.status, kStatusBwdTimeout, kWaitTimeoutNs);
    for (int e = nv - VS < 0 ? 0 : nv - VS; e < nv; ++e)
      mbar_wait(full_v(e % VS), static_cast<uint32_t>(e / VS) & 1u, p.status, kStatusBwdTimeout, kWaitTimeoutNs);
    mbar_wait(bar_q, 0, p.status, kStatusBwdTimeout, kWaitTimeoutNs);
  } else if (warp == 0 && lane == 0 && n > 0) {
    // ============================================================ MMA issuer
    bool ok = bwd_wait(bar_q, 0, p, abort_flag);
    tc_fence_after();
    const uint64_t dq0 = smem_desc(q_smem, 16, 1024, kSwizzle128B);
    const uint64_t do0 = smem_desc(o_smem, 16, 1024, kSwizzle128B);
    // S-type product: d = A (K-major, rows = queries) * B^T (K-major, rows = keys), K = D
    auto issue_qk = [&](uint32_t d, uint64_t a0, int slot) {
      const uint64_t bk = smem_desc(k_smem(slot), 16, 1024, kSwizzle128B);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * L::kChunkBytes + (kk % 4) * 32) >> 4);
        mma_ss(d, a0 + off, bk + off, kIdescS, kk > 0 ? 1u : 0u);
      }
    };
    // dP over the key half `half` (V rows 64 * half.., 8 KB into each 16 KB chunk) into its
    // half of the dP buffer
    auto issue_dp = [&](int slot, int half) {
      const uint64_t bv = smem_desc(v_smem(slot), 16, 1024, kSwizzle128B) + static_cast<uint64_t>((half * 64 * 128) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * L::kChunkBytes + (kk % 4) * 32) >> 4);
        mma_ss(tmem + kDpCol + 64u * half, do0 + off, bv + off, kIdescHalf, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_sdp(half));
    };
    // dQ += dS K over the key half `half`: A = dS, 16-bit pairs in columns
    // [64 * half, 64 * half + 32) of tile t's S buffer
    auto issue_dq = [&](int t, int slotK, int half) {
      const uint64_t bkn = smem_desc(k_smem(slotK), L::kChunkBytes, 1024, kSwizzle128B);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = 4 * half + q;
        mma_ts(tmem + kDqCol, tmem + s_col(t) + 64u * half + 8u * q, bkn + static_cast<uint64_t>((kk * 2048) >> 4),
               kIdescDq, (t > 0 || kk > 0) ? 1u : 0u);
      }
    };
    auto k_wait = [&](int tile) {  // K_tile is in slot tile % KS
      if (!bwd_wait(full_k(tile % KS), static_cast<uint32_t>(tile / KS) & 1u, p, abort_flag)) return false;
      tc_fence_after();
      return true;
    };
    auto v_wait = [&](int tile) {
      if (!bwd_wait(full_v(tile % VS), static_cast<uint32_t>(tile / VS) & 1u, p, abort_flag)) return false;
      tc_fence_after();
      return true;
    };
    // Software-pipelined by key half: once warpgroup A has finished half A of tile t, dQ
    // over that half runs and dP half A of tile t + 1 is formed while warpgroup B still
    // works on half B of tile t; S alternates between two buffers one tile ahead.
    if (ok && k_wait(0)) issue_qk(tmem + s_col(0), dq0, 0);
    else ok = false;
    if (ok && v_wait(0)) {
      issue_dp(0, 0);
      issue_dp(0, 1);
      mma_commit(empty_v(0));
    } else {
      ok = false;
    }
    if (ok && n > 1) {
      if (k_wait(1)) issue_qk(tmem + s_col(1), dq0, 1 % KS);
      else ok = false;
    }
    for (int t = 0; t < n && ok; ++t) {
      const int sK = t % KS, sV1 = (t + 1) % VS;
      if (!bwd_wait(bar_ds(0), static_cast<uint32_t>(t) & 1u, p, abort_flag)) break;
      tc_fence_after();
      issue_dq(t, sK, 0);
      if (t + 1 < n) {
        if (!v_wait(t + 1)) break;
        issue_dp(sV1, 0);  // dP half A of tile t + 1 (S of t + 1 is already issued)
      }
      if (!bwd_wait(bar_ds(1), static_cast<uint32_t>(t) & 1u, p, abort_flag)) break;
      tc_fence_after();
      issue_dq(t, sK, 1);
      mma_commit(empty_k(sK));
      if (t + 1 < n) {
        issue_dp(sV1, 1);
        mma_commit(empty_v(sV1));
      }
      if (t + 2 < n) {
        if (!k_wait(t + 2)) break;
        issue_qk(tmem + s_col(t + 2), dq0, (t + 2) % KS);  // into tile t's buffer, whose dS is consumed
      }
    }
    mma_commit(bar_done);
    mbar_wait(bar_done, 0, p.status, kStatusBwdTimeout, kWaitTimeoutNs);
  } else if (warp >= kBwdWarp0) {
    // ============================================================ element-wise warps
    const int wq = warp & 3;
    const int wg = (warp - kBwdWarp0) >> 2;  // column half of this warpgroup
    const uint32_t cb = 64u * static_cast<uint32_t>(wg);
    const int row = wq * 32 + lane;
    const int i = q0 + row;
    const bool row_valid = i < p.Sq;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const int64_t srow = static_cast<int64_t>(bh) * p.Sq_pad + (row_valid ? i : 0);
    const float nlse2 = row_valid ? p.nlse2[srow] : -INFINITY;
    const uint64_t nd2 = pack2(row_valid ? p.ndelta[srow] : 0.f, row_valid ? p.ndelta[srow] : 0.f);
    const uint64_t sc2 = pack2(p.scale_log2, p.scale_log2);
    float slope2 = 0.f;
    if (SCORE == kScoreAlibi)
      slope2 = (p.slopes ? __ldg(p.slopes + h) : exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(p.H))) *
               kLog2e;
    int64_t row_lo, row_hi, lo_last, hi_first, t0, t1;
    row_interval<MASK>(i, mk, row_lo, row_hi);
    row_interval<MASK>(q1 - 1, mk, lo_last, t1);
    row_interval<MASK>(q0, mk, t0, hi_first);
    bool ok = true;
    auto walk = asc_bits(smem_words, BLOCKS ? n_words : 0);
    for (int t = 0; t < n; ++t) {
      const bool got = bwd_wait(bar_sdp(wg), static_cast<uint32_t>(t) & 1u, p, abort_flag);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int k0 = (BLOCKS ? walk.cur : lo + t) * kBN;
      bool full;
      int64_t keep_lo = row_lo, keep_hi = row_hi;
      if constexpr (BLOCKS) {
        if (walk.cur_full) {  // a FULL block keeps every key below Skv
          keep_lo = 0;
          keep_hi = p.Skv - 1;
        }
        full = row_valid && walk.cur_full && k0 + kBN <= p.Skv;
        walk.advance();
      } else {
        full = row_valid && tile_class_of(lo_last, hi_first, k0, kBN, p.Skv) == kTileFull;
      }
      int c_lo = 0, c_hi = kBN - 1;
      if (!full) {
        col_interval_of(keep_lo, keep_hi, k0, c_lo, c_hi);
        if (!row_valid) {
          c_lo = 1;
          c_hi = 0;
        }
      }
      const uint32_t tS = tmem + lane_off + s_col(t) + cb, tP = tmem + lane_off + kDpCol + cb;
      const float base = slope2 * static_cast<float>(k0 + static_cast<int>(cb) - i) + nlse2;
      const uint64_t nl2 = pack2(nlse2, nlse2);
#pragma unroll
      for (int part = 0; part < 2; ++part) {  // 32 columns at a time
        uint32_t sr[32], pr[32], w[16];
        tmem_ld32(tS + 32u * part, sr);
        tmem_ld32(tP + 32u * part, pr);
        float* x = reinterpret_cast<float*>(sr);
        const int c0 = static_cast<int>(cb) + 32 * part;  // column of x[0] within the tile
        // x = s * scale * log2(e) + bias - LSE * log2(e), two columns per instruction
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = 2 * e;
          const uint64_t b2 = SCORE == kScoreAlibi
                                  ? pack2(fmaf(slope2, static_cast<float>(32 * part + c), base),
                                          fmaf(slope2, static_cast<float>(32 * part + c + 1), base))
                                  : nl2;
          unpack2(fma2(pack2(x[c], x[c + 1]), sc2, b2), x[c], x[c + 1]);
        }
        if (!full) {  // warp-uniform: the mask pass runs on PARTIAL tiles only
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c0 + c < c_lo || c0 + c > c_hi) x[c] = -INFINITY;
        }
        // branch-free: ex2(-inf) = 0 gives dS = 0 for dropped keys; dS = P (dP - delta)
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint64_t p2 = pack2(ex2_approx(x[2 * e]), ex2_approx(x[2 * e + 1]));
          float d0, d1;
          unpack2(mul2(p2, add2(pack2(__uint_as_float(pr[2 * e]), __uint_as_float(pr[2 * e + 1])), nd2)), d0, d1);
          w[e] = DtypeBits<T>::pack(d0, d1);
        }
        tmem_st16(tS + 16u * part, w);  // columns cb + [0, 32): read by this warpgroup already
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_ds(wg));
    }
    // epilogue: dQ row * scale
    bool ran = ok && n > 0;
    if (ran) {
      const bool got = bwd_wait(bar_done, 0, p, abort_flag);
      if (!__all_sync(0xffffffffu, got)) ran = false;
      tc_fence_after();
    }
    T* out = reinterpret_cast<T*>(p.dq) + (static_cast<int64_t>(bh) * p.Sq + i) * D;
#pragma unroll 1
    for (int c = wg * (D / 2); c < (wg + 1) * (D / 2); c += 32) {  // each warpgroup half of the columns
      uint32_t r[32];
      if (ran) tmem_ld32(tmem + lane_off + kDqCol + c, r);
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        w[e] = DtypeBits<T>::pack(ran ? __uint_as_float(r[2 * e]) * p.scale : 0.f,
                                  ran ? __uint_as_float(r[2 * e + 1]) * p.scale : 0.f);
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
        for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK, dV

template <int D, typename T, int SCORE, int MASK, bool BLOCKS>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const BwdParams p) {
  using L = BwdDkvSmem<D>;
  constexpr int NS = L::kSlots;
  constexpr int kChunks = D / 64;
  constexpr uint32_t kIdescHalf = idesc_f16(DtypeBits<T>::kFmt, kBN, kBM / 2, 0);  // S^T, dP^T halves
  constexpr uint32_t kIdescAcc = idesc_f16(DtypeBits<T>::kFmt, kBN, D, 1);  // dV, dK: N-major B
  constexpr bool kDoc = is_doc_mask(MASK);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t sbase = (raw_addr + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_addr);
  const uint32_t bar_kv = sbase + L::kBarOff;
  auto bar_full = [&](int s) { return sbase + L::kBarOff + 8u * (1 + s); };
  auto bar_empty = [&](int s) { return sbase + L::kBarOff + 8u * (1 + NS + s); };
  const uint32_t bar_sdp0 = sbase + L::kBarOff + 8u * (1 + 2 * NS);
  auto bar_sdp = [&](int half) { return bar_sdp0 + 8u * half; };
  auto bar_pds = [&](int half) { return bar_sdp0 + 8u * (2 + half); };
  const uint32_t bar_done = bar_sdp0 + 32u;
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sgen + L::kTmemPtrOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kTmemPtrOff + 4);
  const uint32_t k_smem = sbase + L::kKOff, v_smem = k_smem + L::kTileBytes;
  auto slot_base = [&](int s) { return static_cast<uint32_t>(L::kSlotOff + s * L::kSlotBytes); };
  auto q_slot = [&](int s) { return sbase + slot_base(s); };
  auto o_slot = [&](int s) { return sbase + slot_base(s) + L::kTileBytes; };
  auto stat_slot = [&](int s) { return slot_base(s) + 2 * L::kTileBytes; };  // byte offset from sbase

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int kt, bkv;
  unit_coords_of(static_cast<int>(blockIdx.x), p.n_ktiles, p.kv_group, p.B * p.Hkv, bkv, kt);
  kt = p.n_ktiles - 1 - kt;  // ascending: under causal masks the first key tiles see the most queries
  const int hk = bkv % p.Hkv, b = bkv / p.Hkv;
  const int k0 = kt * kBN;
  MaskArgs mk = p.mask;
  if constexpr (kDoc) {
    mk.off_q += static_cast<int64_t>(b) * (mk.n_docs + 1);
    mk.off_kv += static_cast<int64_t>(b) * (mk.n_docs + 1);
  }
  // does query tile t see key tile kt?
  auto active = [&](int t) {
    int lo, hi;
    tile_range<MASK>(t * kBM, min(t * kBM + kBM, p.Sq), kBN, mk, lo, hi);
    return kt >= lo && kt < hi;
  };
  // steps: (query head of the group) x (active query tile); every role walks the same list.
  // Block mask: the steps are the set bits of this key tile's transposed bitmap (pairs
  // hg * n_qtiles + t in ascending order, hg major), with the FULL bitmap alongside.
  const uint32_t* tb_row =
      BLOCKS ? p.tbits + ((static_cast<int64_t>(b) * p.Hkv + hk) * p.n_ktiles + kt) * 2 * p.tb_words : nullptr;
  const int tb_words = p.tb_words;
  auto tb_load = [tb_row, tb_words](int w, int which) { return __ldg(tb_row + which * tb_words + w); };
  int n = 0;
  if constexpr (BLOCKS) {
    for (int w = 0; w < p.tb_words; ++w) n += __popc(tb_load(w, 0));
  } else {
    int n_active = 0;
    for (int t = 0; t < p.n_qtiles; ++t) n_active += active(t) ? 1 : 0;
    n = n_active * p.G;
  }
  // calls f(hg, t, listed_full) for every step in order; f returns false to stop
  auto for_steps = [&](auto&& f) {
    if constexpr (BLOCKS) {
      for (auto w = asc_bits(tb_load, p.tb_words); w.cur >= 0; w.advance())
        if (!f(w.cur / p.n_qtiles, w.cur % p.n_qtiles, w.cur_full)) return;
    } else {
      for (int hg = 0; hg < p.G; ++hg)
        for (int t = 0; t < p.n_qtiles; ++t)
          if (active(t) && !f(hg, t, false)) return;
    }
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_sdp(0), 1);
    mbar_init(bar_sdp(1), 1);
    mbar_init(bar_pds(0), kBN);
    mbar_init(bar_pds(1), kBN);
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_ptr), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  // TMEM columns: S^T / P^T [0,128), dP^T / dS^T [128,256), dV [256, 256+D), dK [256+D, 256+2D)
  constexpr uint32_t kSCol = 0, kDpCol = 128, kDvCol = 256, kDkCol = 256 + D;

  if (warp == 1 && lane == 0 && n > 0) {
    // ============================================================ TMA producer
    mbar_arrive_expect_tx(bar_kv, 2 * L::kTileBytes);
    for (int c = 0; c < kChunks; ++c) {
      tma_load_3d(k_smem + c * L::kChunkBytes, &tmK, bar_kv, c * 64, k0, bkv);
      tma_load_3d(v_smem + c * L::kChunkBytes, &tmV, bar_kv, c * 64, k0, bkv);
    }
    int u = 0;
    for_steps([&](int hg, int t, bool) -> bool {
      const int bh = b * p.H + hk * p.G + hg;
      const int s = u % NS;
      if (!bwd_wait(bar_empty(s), (static_cast<uint32_t>(u / NS) & 1u) ^ 1u, p, abort_flag)) return false;
      mbar_arrive_expect_tx(bar_full(s), 2 * L::kTileBytes + L::kStatBytes);
      for (int c = 0; c < kChunks; ++c) {
        tma_load_3d(q_slot(s) + c * L::kChunkBytes, &tmQ, bar_full(s), c * 64, t * kBM, bh);
        tma_load_3d(o_slot(s) + c * L::kChunkBytes, &tmO, bar_full(s), c * 64, t * kBM, bh);
      }
      const int64_t srow = static_cast<int64_t>(bh) * p.Sq_pad + t * kBM;
      bulk_load(sbase + stat_slot(s), p.nlse2 + srow, kBM * 4, bar_full(s));
      bulk_load(sbase + stat_slot(s) + kBM * 4, p.ndelta + srow, kBM * 4, bar_full(s));
      ++u;
      return true;
    });
    for (int e = u - NS < 0 ? 0 : u - NS; e < u; ++e)
      mbar_wait(bar_full(e % NS), static_cast<uint32_t>(e / NS) & 1u, p.status, kStatusBwdTimeout, kWaitTimeoutNs);
    mbar_wait(bar_kv, 0, p.status, kStatusBwdTimeout, kWaitTimeoutNs);
  } else if (warp == 0 && lane == 0 && n > 0) {
    // ============================================================ MMA issuer
    bool ok = bwd_wait(bar_kv, 0, p, abort_flag);
    tc_fence_after();
    const uint64_t dk0 = smem_desc(k_smem, 16, 1024, kSwizzle128B);
    const uint64_t dv0 = smem_desc(v_smem, 16, 1024, kSwizzle128B);
    // S^T and dP^T for the query half `half` (64 queries: rows 64 * half.. of the Q / dO
    // tiles, 8 KB into each 16 KB chunk) of step u's slot, into their half of the buffers
    auto issue_sdp = [&](int s, int half) {
      const uint64_t hoff = static_cast<uint64_t>((half * 64 * 128) >> 4);
      const uint64_t bq = smem_desc(q_slot(s), 16, 1024, kSwizzle128B) + hoff;
      const uint64_t bo = smem_desc(o_slot(s), 16, 1024, kSwizzle128B) + hoff;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * L::kChunkBytes + (kk % 4) * 32) >> 4);
        mma_ss(tmem + kSCol + 64u * half, dk0 + off, bq + off, kIdescHalf, kk > 0 ? 1u : 0u);   // S^T = K Q^T
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk / 4) * L::kChunkBytes + (kk % 4) * 32) >> 4);
        mma_ss(tmem + kDpCol + 64u * half, dv0 + off, bo + off, kIdescHalf, kk > 0 ? 1u : 0u);  // dP^T = V dO^T
      }
      mma_commit(bar_sdp(half));
    };
    // dV += P^T dO and dK += dS^T Q over the query half `half` (A = 16-bit pairs in
    // columns [64 * half, 64 * half + 32) of the S^T and dP^T buffers)
    auto issue_acc = [&](int s, int u, int half) {
      const uint64_t bon = smem_desc(o_slot(s), L::kChunkBytes, 1024, kSwizzle128B);
      const uint64_t bqn = smem_desc(q_slot(s), L::kChunkBytes, 1024, kSwizzle128B);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int kk = 4 * half + q;
        const uint64_t off = static_cast<uint64_t>((kk * 2048) >> 4);
        const uint32_t acol = 64u * half + 8u * q;
        mma_ts(tmem + kDvCol, tmem + kSCol + acol, bon + off, kIdescAcc, (u > 0 || kk > 0) ? 1u : 0u);
        mma_ts(tmem + kDkCol, tmem + kDpCol + acol, bqn + off, kIdescAcc, (u > 0 || kk > 0) ? 1u : 0u);
      }
    };
    // Software-pipelined by query half: as soon as warpgroup A has finished half A of step
    // u, its products run and half A of step u + 1 is formed, while warpgroup B still works
    // on half B of step u (the halves use disjoint TMEM columns).
    if (ok && bwd_wait(bar_full(0), 0, p, abort_flag)) {
      tc_fence_after();
      issue_sdp(0, 0);
      issue_sdp(0, 1);
    } else {
      ok = false;
    }
    for (int u = 0; u < n && ok; ++u) {
      const int s = u % NS, s1 = (u + 1) % NS;
      const bool more = u + 1 < n;
      if (!bwd_wait(bar_pds(0), static_cast<uint32_t>(u) & 1u, p, abort_flag)) break;
      tc_fence_after();
      issue_acc(s, u, 0);
      if (more) {
        if (!bwd_wait(bar_full(s1), static_cast<uint32_t>((u + 1) / NS) & 1u, p, abort_flag)) break;
        tc_fence_after();
        issue_sdp(s1, 0);
      }
      if (!bwd_wait(bar_pds(1), static_cast<uint32_t>(u) & 1u, p, abort_flag)) break;
      tc_fence_after();
      issue_acc(s, u, 1);
      mma_commit(bar_empty(s));
      if (more) issue_sdp(s1, 1);
    }
    mma_commit(bar_done);
    mbar_wait(bar_done, 0, p.status, kStatusBwdTimeout, kWaitTimeoutNs);
  } else if (warp >= kBwdWarp0) {
    // ============================================================ element-wise warps
    const int wq = warp & 3;
    const int wg = (warp - kBwdWarp0) >> 2;  // column (query) half of this warpgroup
    const int cb = 64 * wg;
    const int row = wq * 32 + lane;
    const int j = k0 + row;  // this thread's key
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    int64_t key_lo, key_hi;
    key_interval<MASK>(j, mk, p.Sq, key_lo, key_hi);
    const uint64_t sc2 = pack2(p.scale_log2, p.scale_log2);
    bool ok = true;
    int u = 0;
    int slope_h = -1;
    float slope2 = 0.f;
    for_steps([&](int hg, int t, bool listed_full) -> bool {
      {
        const int h = hk * p.G + hg;
        if (SCORE == kScoreAlibi && h != slope_h) {
          slope_h = h;
          slope2 = (p.slopes ? __ldg(p.slopes + h)
                             : exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(p.H))) *
                   kLog2e;
        }
        const int s = u % NS;
        // S^T / dP^T ready; the slot's statistics (written by the bulk copy) are read
        // below, so observe the slot's own barrier too
        const bool got = bwd_wait(bar_sdp(wg), static_cast<uint32_t>(u) & 1u, p, abort_flag) &&
                         bwd_wait(bar_full(s), static_cast<uint32_t>(u / NS) & 1u, p, abort_flag);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          return false;
        }
        tc_fence_after();
        const int q0 = t * kBM;
        // a FULL block keeps every query (rows past Sq have P = 0 through their -inf LSE)
        const bool full = BLOCKS ? listed_full : tile_class<MASK>(q0, min(q0 + kBM, p.Sq), k0, kBN, mk) == kTileFull;
        int c_lo = 0, c_hi = kBM - 1;
        if (!full) col_interval_of(key_lo, key_hi, q0, c_lo, c_hi);
        const float* stat = reinterpret_cast<const float*>(sgen + stat_slot(s));
        const float base = slope2 * static_cast<float>(j - q0 - cb);
#pragma unroll
        for (int part = 0; part < 2; ++part) {  // 32 columns (queries) at a time
          const int c0 = cb + 32 * part;       // column of x[0] within the tile
          uint32_t sr[32], pr[32], wp[16], wd[16];
          tmem_ld32(tmem + lane_off + kSCol + c0, sr);
          tmem_ld32(tmem + lane_off + kDpCol + c0, pr);
          float* x = reinterpret_cast<float*>(sr);
          const uint64_t* nl = reinterpret_cast<const uint64_t*>(stat + c0);  // -lse2 pairs
          // x = s * scale * log2(e) + bias - LSE * log2(e), two columns per instruction
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = 2 * e;
            uint64_t b2 = nl[e];
            if (SCORE == kScoreAlibi)
              b2 = add2(b2, pack2(fmaf(-slope2, static_cast<float>(32 * part + c), base),
                                  fmaf(-slope2, static_cast<float>(32 * part + c + 1), base)));
            unpack2(fma2(pack2(x[c], x[c + 1]), sc2, b2), x[c], x[c + 1]);
          }
          if (!full) {  // warp-uniform: the mask pass runs on PARTIAL tiles only
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c0 + c < c_lo || c0 + c > c_hi) x[c] = -INFINITY;
          }
          const uint64_t* nd = reinterpret_cast<const uint64_t*>(stat + kBM + c0);  // -delta pairs
          // dS = P (dP - delta), two columns per instruction
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = ex2_approx(x[2 * e]), p1 = ex2_approx(x[2 * e + 1]);
            wp[e] = DtypeBits<T>::pack(p0, p1);
            float d0, d1;
            unpack2(mul2(pack2(p0, p1), add2(pack2(__uint_as_float(pr[2 * e]), __uint_as_float(pr[2 * e + 1])), nd[e])),
                    d0, d1);
            wd[e] = DtypeBits<T>::pack(d0, d1);
          }
          // columns cb + [0, 32) of each buffer, already read by this warpgroup
          tmem_st16(tmem + lane_off + kSCol + cb + 16u * part, wp);
          tmem_st16(tmem + lane_off + kDpCol + cb + 16u * part, wd);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_pds(wg));
        ++u;
      }
      return true;
    });
    // epilogue: dK = scale * (dS^T Q), dV = P^T dO
    bool ran = ok && n > 0;
    if (ran) {
      const bool got = bwd_wait(bar_done, 0, p, abort_flag);
      if (!__all_sync(0xffffffffu, got)) ran = false;
      tc_fence_after();
    }
    const bool key_valid = j < p.Skv;
    const int64_t orow = (static_cast<int64_t>(bkv) * p.Skv + j) * D;
    {
      const int which = wg;  // warpgroup 0 writes dV, warpgroup 1 dK
      T* out = reinterpret_cast<T*>(which ? p.dk : p.dv) + orow;
      const float mul = which ? p.scale : 1.0f;
      const uint32_t col = which ? kDkCol : kDvCol;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t r[32];
        if (ran) tmem_ld32(tmem + lane_off + col + c, r);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = DtypeBits<T>::pack(ran ? __uint_as_float(r[2 * e]) * mul : 0.f,
                                    ran ? __uint_as_float(r[2 * e + 1]) * mul : 0.f);
        if (key_valid) {
          uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
          for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace flexattn
