// flex_fwd_sm100.cuh -- flex-attention forward kernel for sm_100a.
//
// Computes, per query row i of (batch b, head h),
//   O = softmax(mask_mod(score_mod(scale * Q K^T))) V  and  LSE = log-sum-exp (natural log),
// following FlyDSL PR 931 "Add flex_attention (score_mod / mask_mod) on the generic
// flash-attention kernel", Summary (score_mod sees the scaled score and runs before the
// mask; fully masked rows give O = 0 / LSE = -inf) with the hooks chosen at compile time,
// so the no-mod instantiation carries no hook code at all.
//
// One CTA owns two 128-row query tiles of one (b, h) and walks the key/value tiles both
// of them need.  Three warpgroups:
//   warp 0      MMA issuer (one thread): S_k = Q_k K_j^T and O_k += P_k V_j with tcgen05,
//               accumulators in tensor memory.  It is warp 0 so that the warp scheduler of
//               its sub-partition, shared with two busy softmax warps, serves it first.
//               A block-mask CTA whose steps often visit one query tile only takes a
//               second issuer in warp 2: warp 0 then issues for query tile 0 and warp 2
//               for tile 1 (kTwoIssuerShare below).
//   warp 1      TMA producer: Q tiles once, then K_j, V_j into a ring of shared-memory slots
//   warps 2-3   idle (they only give their registers to the softmax warpgroups)
//   warps 4-7   softmax for query tile 0, warps 8-11 for query tile 1: each thread owns one
//               query row (= one TMEM lane), reads its S row from TMEM, applies score_mod,
//               mask (PARTIAL tiles only) and the online base-2 softmax, writes P (16-bit)
//               back into TMEM over S in two 64-column halves (each signalled on its own
//               barrier so the P.V matmul can start on the first half), rescales its O row
//               when the running max grows by more than 2^8, and finally normalises O and
//               writes O and LSE.  kEmuPairsPerHalf of each 32 column pairs can evaluate
//               2^x as a polynomial on the FMA pipe instead of the MUFU unit.
// With a block mask (the BLOCKS instantiations) each query tile visits the key tiles its
// partial and full lists name instead of the range its mask_mod implies; the CTA walks the
// union of its two tiles' sets, and a tile absent from one set is simply not issued for
// that query tile.  The sets live in shared memory as bitmaps built at the start.
// Key tiles are visited from the last to the first.  With t counting steps, the MMA order
// S0(t0) S1(t0) | PV0(t) S0(t+1) PV1(t) S1(t+1) | ... lets one softmax warpgroup work
// while the tensor core runs the other tile's matmuls.  With two issuers each runs
// S_k(t0) | PV_k(t) S_k(t+1) | ... for its tile; a K/V slot is then freed when both have
// arrived on its empty barrier (count 2), and an issuer whose tile skips a step still
// waits for that step's slots to be filled before it arrives, so it can never arrive for
// a slot's next use before the other issuer has arrived for the current one.
//
// Tensor memory (512 columns x 128 lanes): S0 [0,128) S1 [128,256) O0 [256,256+D)
// O1 [384,384+D); P_k aliases the first 64 columns of S_k (two 16-bit values per column).
// Shared memory: Q0, Q1 and NS key/value slots, each a 128-row tile stored as D/64 chunks
// of [128 rows x 128 bytes] in the 128-byte swizzled layout TMA writes and the tensor
// core reads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>

#include "mask_rules.cuh"
#include "ptx_sm100.cuh"

namespace flexattn {

constexpr int kBM = 128;        // query rows per tile (tcgen05 M)
constexpr int kBN = 128;        // keys per tile
constexpr int kFwdThreads = 384;
constexpr int kMmaWarp = 0;   // issuer of query tile 0
constexpr int kMmaWarp1 = 2;  // issuer of query tile 1
constexpr int kTmaWarp = 1;
constexpr int kSoftmaxWarp0 = 4;        // warps 4-7: query tile 0, warps 8-11: query tile 1
constexpr uint32_t kSoftmaxRegs = 200;  // per thread, softmax warpgroups after setmaxnreg
constexpr uint32_t kAuxRegs = 96;       // per thread, producer/MMA warpgroup after setmaxnreg
// 256 * 200 + 128 * 96 = 63488 <= 384 * 168 (the launch allotment at 384 threads); per
// SM sub-partition (one warp of each warpgroup) 200 + 200 + 96 <= 512
static_assert(256 * kSoftmaxRegs + 128 * kAuxRegs <= (65536 / kFwdThreads) / 8 * 8 * kFwdThreads,
              "setmaxnreg split exceeds the registers the block is launched with");
static_assert(2 * kSoftmaxRegs + kAuxRegs <= 512, "per sub-partition register file exceeded");
// Of the 32 column pairs of each 64-column half, how many take 2^x from the polynomial on
// the FMA pipe instead of MUFU ex2 (spread evenly over the half).  Measured on B200 at
// D = 128: 4 of 32 cost 13 %, 8 of 32 cost 19 % on dense work, so none by default.
#ifndef FLEX_FWD_EMU_PAIRS
#define FLEX_FWD_EMU_PAIRS 0
#endif
constexpr int kEmuPairsPerHalf = FLEX_FWD_EMU_PAIRS;
__host__ __device__ constexpr bool emu_pair(int i) { return (i * kEmuPairsPerHalf) % 32 < kEmuPairsPerHalf; }
// MMA issuers: one thread for both query tiles, or one per tile.  One issuer finishes a
// tile's P.V and its next S back to back, which keeps each softmax warpgroup's wait for
// its next S short; two issuers interleave both tiles' products and hide each other's
// barrier probes, which pays when many steps visit one tile only.  Measured on B200 (B2
// H32 S8192): two issuers are 35 % slower on dense work and 21 % slower on causal block
// lists, 10-20 % faster on random half-dense block lists.  So analytic masks always use
// one issuer, and a block-mask CTA takes two when at least a third of its steps visit
// only one of its two query tiles (decided per CTA from its visit bitmaps).
constexpr int kTwoIssuerShare = 3;  // two issuers iff kTwoIssuerShare * single-tile steps >= steps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O when the max grows > 2^8
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr unsigned kStatusFwdTimeout = 2u;
// Block mask: key tiles a bitmap can name (Skv <= 2048 * 128), and its size in words.
constexpr int kMaxBlockKeyTiles = 2048;
constexpr int kBlkWords = kMaxBlockKeyTiles / 32;
// A FULL-listed key tile that runs past Skv: only the key-length rule masks it.
constexpr int kTileFullRagged = 3;
// Most parts the persistent kernel splits one unit's key ranges into (FwdParams::n_parts).
constexpr int kMaxParts = 4;

// Step record: what the MMA issuer does at one step of the CTA's walk over key tiles.
// The TMA producer, which walks the same tiles ahead of time, writes the record of step
// t + 1 before it signals V of step t, so the issuer never walks the sets itself.
constexpr uint32_t kRecIn0 = 1u << 0;    // query tile 0 visits this key tile
constexpr uint32_t kRecIn1 = 1u << 1;
constexpr uint32_t kRecPre0 = 1u << 2;   // ... and its next key tile is the next step's
constexpr uint32_t kRecPre1 = 1u << 3;
constexpr uint32_t kRecLast0 = 1u << 4;  // ... and this is its last key tile
constexpr uint32_t kRecLast1 = 1u << 5;
constexpr uint32_t kRecEnd = 1u << 6;    // no step: the walk is over
constexpr uint32_t kRecNewItem = 1u << 7;  // persistent kernel: the first step of the next item

struct FwdParams;
__device__ __forceinline__ void unit_coords(const FwdParams& p, int unit, int& bh, int& pair);

struct FwdParams {
  void* o;
  float* lse;
  uint8_t* tile_map;   // debug tile map or nullptr
  unsigned* status;    // device status word
  int H, Hkv, G, Sq, Skv;
  int n_qtiles, n_ktiles, n_pairs;
  int n_units;         // B * H * n_pairs (the persistent kernel loops over them)
  int bh_total;        // B * H
  int head_group;      // units run in groups of head_group heads (unit_coords)
  int persist_grid;    // CTAs of the persistent kernel (0: one CTA per unit)
  // Persistent kernel: items [0, n_full) are whole units; items [n_full, n_items) split
  // the last n_units - n_full units' key ranges into n_parts parts each.  The parts of a
  // (unit, tile, warp) but the last to arrive leave their unnormalised O and (max, sum)
  // per row in part_o / part_ml; the last merges them.  The counters are tagged
  // (tagged_add): every launch brings a new part_tag, so they are never zeroed.
  int n_full, n_parts, n_items;
  float* part_o;       // [split units][n_parts][2 tiles][D / 4][kBM rows] float4 (fp32 O)
  float2* part_ml;     // [split units][n_parts][2 tiles][kBM rows] (max in log2 units, sum)
  unsigned long long* part_cnt;  // [split units][2 tiles][4 warps][arrived, ready]
  unsigned part_tag;
  float scale_log2;    // scale * log2(e)
  const float* slopes; // alibi: captured per-head slopes [H], or nullptr for 2^(-8(h+1)/H)
  MaskArgs mask;       // document rules: boundaries of batch 0, advanced per batch below
  // Block mask (BLOCKS instantiations): [0] partial lists, [1] full lists; counts are
  // [rows x n_qtiles], indices [rows x n_qtiles x blk_max]; row of (b, h) =
  // b * blk_b_stride + h * blk_h_stride (a stride of 0 shares one row).
  const int32_t* blk_num[2];
  const int32_t* blk_idx[2];
  int blk_max;
  int blk_b_stride, blk_h_stride;
};

// unit -> (b * H + h, pair of query tiles).  Heads run in groups of head_group; within a
// group the pairs run from the last to the first (under causal masks the heaviest first),
// each pair over all the group's heads, so that the block scheduler's last wave holds the
// lightest units while the group's K/V stay in L2.  head_group = 1: head by head.
__device__ __forceinline__ void unit_coords_of(int unit, int n_pairs, int head_group, int bh_total, int& bh,
                                               int& pair) {
  const int per_group = head_group * n_pairs;
  const int gi = unit / per_group;
  const int base = gi * head_group;
  const int gh = min(head_group, bh_total - base);  // heads in this group
  const int r = unit - gi * per_group;
  pair = n_pairs - 1 - r / gh;
  bh = base + r % gh;
}
__device__ __forceinline__ void unit_coords(const FwdParams& p, int unit, int& bh, int& pair) {
  unit_coords_of(unit, p.n_pairs, p.head_group, p.bh_total, bh, pair);
}


// Block-mask / document bitmaps: full0, full1, act0, act1, and with both a block mask
// and a document mask the document sets doc0, doc1 (kBlkWords words each).
constexpr int fwd_bitmaps(bool blocks, bool doc) { return blocks ? (doc ? 6 : 4) : (doc ? 4 : 0); }

template <int D, bool BLOCKS = false, bool DOC = false>
struct FwdSmem {
  static constexpr int kTileBytes = kBM * D * 2;          // one 128-row tile
  static constexpr int kChunkBytes = kBM * 128;           // one 64-element-wide chunk
  // Key/value ring depth.  K_j and V_j take consecutive entries; K_j is released as soon
  // as both S_k(j) are issued, V_j only after both P_k V_j, so with 5 slots V_{j+2} waits
  // on K_j rather than on V_j and gets about two tile steps of load lead time.
  static constexpr int kSlots = D == 128 ? 5 : 12;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kSlots * kTileBytes;
  // barriers: q, full[NS], empty[NS], s_full[2], p_half[2][2], o_full[2], drain[2], q_free;
  // then the tmem address
  static constexpr int kNumBars = 1 + 2 * kSlots + 2 + 4 + 2 + 2 + 1;
  static constexpr int kTmemPtrOff = kBarOff + kNumBars * 8;
  // step records (kRec*): one per key/value slot, plus the first step's
  static constexpr int kRecOff = kTmemPtrOff + 16;
  static constexpr int kRecBytes = ((kSlots + 1) * 4 + 15) / 16 * 16;
  // document rules: the documents of each tile's first and last row (4 ints)
  static constexpr int kDocOff = kRecOff + kRecBytes;
  static constexpr int kBlkOff = kDocOff + (DOC ? 16 : 0);
  static constexpr int kBytes = kBlkOff + fwd_bitmaps(BLOCKS, DOC) * kBlkWords * 4;
  static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024 bytes
  static_assert(kAlloc <= 227 * 1024, "shared memory per CTA exceeded");
};

template <typename T>
struct DtypeBits;
template <>
struct DtypeBits<__nv_bfloat16> {
  static constexpr uint32_t kFmt = 1;
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};
template <>
struct DtypeBits<__half> {
  static constexpr uint32_t kFmt = 0;
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
};

// Walk of the key tiles one query tile visits, from the last to the first.  cur is the
// current tile (-1 once the walk is over), advance() moves to the next one.
//
// BitCursor walks the set bits of a shared-memory bitmap with the current 32-bit word in
// a register, so a step costs a few ALU operations and one shared-memory load per 32
// tiles; the companion bitmap (the FULL tiles) is read alongside into cur_full.
struct BitCursor {
  const uint32_t* set;
  const uint32_t* comp;
  int wi;
  uint32_t bits, cword;
  int cur;
  bool cur_full;
  __device__ __forceinline__ void advance() {
    while (bits == 0) {
      if (--wi < 0) {
        cur = -1;
        return;
      }
      bits = set[wi];
      cword = comp[wi];
    }
    const int bit = 31 - __clz(bits);
    bits &= ~(1u << bit);
    cur = (wi << 5) + bit;
    cur_full = (cword >> bit) & 1u;
  }
  // n_tiles <= kMaxBlockKeyTiles; bits at or above n_tiles are clear.
  __device__ __forceinline__ BitCursor(const uint32_t* s, const uint32_t* c, int n_tiles)
      : set(s), comp(c), wi((n_tiles + 31) >> 5), bits(0), cword(0), cur(-1), cur_full(false) {
    advance();
  }
};

// RangeCursor walks the contiguous range [lo, hi) that a mask_mod implies.
struct RangeCursor {
  int lo, cur;
  bool cur_full = false;
  __device__ __forceinline__ RangeCursor(int l, int h) : lo(l), cur(h - 1 >= l ? h - 1 : -1) {}
  __device__ __forceinline__ void advance() { cur = cur - 1 >= lo ? cur - 1 : -1; }
};

__device__ __forceinline__ bool bits_has(const uint32_t* w, int j) { return (w[j >> 5] >> (j & 31)) & 1u; }

// Sets bits [u_lo, u_hi] of a bitmap (word-wise atomic ORs).
__device__ __forceinline__ void bits_set_range(uint32_t* w, int u_lo, int u_hi) {
  for (int wi = u_lo >> 5; wi <= (u_hi >> 5); ++wi) {
    const int a = max(u_lo, wi << 5) & 31, b = min(u_hi, (wi << 5) + 31) & 31;
    const uint32_t m = (b == 31 ? 0xffffffffu : ((2u << b) - 1u)) & ~((1u << a) - 1u);
    atomicOr(w + wi, m);
  }
}

constexpr bool is_doc_mask(int mask) { return mask == kMaskDocument || mask == kMaskDocumentCausal; }

// Block lists as the forward kernels take them: [0] partial, [1] full; counts
// [rows x n_qtiles], indices [rows x n_qtiles x max]; the row of (b, h) is
// b * b_stride + h * h_stride (a stride of 0 shares one row).
struct VisitLists {
  const int32_t* num[2];
  const int32_t* idx[2];
  int max, b_stride, h_stride;
};

// Bitmaps of the visit sets in shared memory (kBlkWords words each): full_k = the key tiles
// query tile k (= 2 * pair + k) keeps whole, act_k = every key tile it visits, and with a
// block mask and a document mask both, doc_k = the tiles its documents reach.
__device__ __forceinline__ uint32_t* visit_full_bits(uint32_t* blk, int k) { return blk + k * kBlkWords; }
__device__ __forceinline__ uint32_t* visit_act_bits(uint32_t* blk, int k) { return blk + (2 + k) * kBlkWords; }

// The visit sets of a CTA's two query tiles (all threads of the CTA call it; it ends
// with the sets complete after a barrier of the caller's).  Document masks build them
// from the documents the tiles' rows span; block masks from the tiles' two lists (with
// a document mask as well, filtered by the document sets); a partial block the mask_mod
// drops whole is left out and one it keeps whole counts as full, so lists read off the
// analytic tile map reproduce the analytic kernel exactly.  lo/hi: the analytic key-tile
// ranges (mask rules other than the document ones).
template <int MASK, bool BLOCKS>
__device__ __forceinline__ void build_visit_sets(uint32_t* blk, int* doc_rows, const VisitLists& bl, int pair,
                                                 int b, int h, const int (&q0)[2], const int (&q1)[2],
                                                 const int (&lo)[2], const int (&hi)[2], const MaskArgs& mk,
                                                 int n_qtiles, int n_ktiles, int Skv) {
  constexpr bool kDoc = MASK == kMaskDocument || MASK == kMaskDocumentCausal;
  auto sel = [](const int (&a)[2], int k) { return k ? a[1] : a[0]; };
  auto full_bits = [&](int k) { return visit_full_bits(blk, k); };
  auto act_bits = [&](int k) { return visit_act_bits(blk, k); };
  auto doc_bits = [&](int k) { return BLOCKS ? blk + (4 + k) * kBlkWords : blk + (2 + k) * kBlkWords; };
  {
    for (int w = threadIdx.x; w < fwd_bitmaps(BLOCKS, kDoc) * kBlkWords; w += kFwdThreads) blk[w] = 0u;
    if constexpr (kDoc) {
      if (threadIdx.x < 4) {  // four independent binary searches, one per lane
        const int k = threadIdx.x >> 1, qt = 2 * pair + k;
        doc_rows[threadIdx.x] =
            qt < n_qtiles ? doc_floor(mk.off_q, mk.n_docs, (threadIdx.x & 1) ? sel(q1, k) - 1 : sel(q0, k)) : -1;
      }
    }
    __syncthreads();
    // Document rules: tile k's class bounds (the first row's last key, the last row's
    // first key); FULL iff lo_last <= k0 and k1 - 1 <= hi_first.
    int64_t lo_last[2] = {0, 0}, hi_first[2] = {-1, -1};
    if constexpr (kDoc) {
      constexpr bool kCausal = MASK == kMaskDocumentCausal;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (2 * pair + k >= n_qtiles) continue;
        int64_t t;
        doc_interval(mk, doc_rows[2 * k + 1], sel(q1, k) - 1, kCausal, lo_last[k], t);
        doc_interval(mk, doc_rows[2 * k], sel(q0, k), kCausal, t, hi_first[k]);
      }
      // every document with rows in tile k: the key tiles those rows keep
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        if (2 * pair + k >= n_qtiles) continue;
        const int d0 = max(doc_rows[2 * k], 0), d1 = min(doc_rows[2 * k + 1], mk.n_docs - 1);
        for (int d = d0 + threadIdx.x; d <= d1; d += kFwdThreads) {
          const int64_t r0 = max(static_cast<int64_t>(sel(q0, k)), static_cast<int64_t>(__ldg(mk.off_q + d)));
          const int64_t r1 = min(static_cast<int64_t>(sel(q1, k)), static_cast<int64_t>(__ldg(mk.off_q + d + 1)));
          if (r0 >= r1) continue;  // no row of this document in the tile
          int64_t a, e;
          doc_interval(mk, d, r1 - 1, kCausal, a, e);  // the union of its rows' intervals
          if (a > e) continue;
          bits_set_range(doc_bits(k), static_cast<int>(a / kBN), static_cast<int>(e / kBN));
        }
        if (!BLOCKS && threadIdx.x == 0) {
          const int64_t f_lo = (lo_last[k] + kBN - 1) / kBN, f_hi = (hi_first[k] + 1) / kBN - 1;
          if (f_lo <= f_hi) bits_set_range(full_bits(k), static_cast<int>(f_lo), static_cast<int>(f_hi));
        }
      }
      if constexpr (BLOCKS) __syncthreads();  // the document sets filter the lists below
    }
    if constexpr (BLOCKS) {
      const int64_t row0 = static_cast<int64_t>(b) * bl.b_stride + static_cast<int64_t>(h) * bl.h_stride;
      // list l = 2 * k + f: query tile 2 * pair + k, f = 0 partial / 1 full (selects, not
      // indexing, so that nothing here is forced into local memory)
      auto count = [&](int k, int f) {
        const int qt = 2 * pair + k;
        const int32_t* num = f ? bl.num[1] : bl.num[0];
        const int c = (qt < n_qtiles && num != nullptr) ? num[row0 * n_qtiles + qt] : 0;
        return c < 0 ? 0 : (c > bl.max ? bl.max : c);
      };
      const int c00 = count(0, 0), c01 = count(0, 1), c10 = count(1, 0), c11 = count(1, 1);
      for (int e = threadIdx.x; e < 4 * bl.max; e += kFwdThreads) {
        const int l = e / bl.max, c = e - l * bl.max;
        const int k = l >> 1, f = l & 1;
        const int cl = k ? (f ? c11 : c10) : (f ? c01 : c00);
        if (c >= cl) continue;
        const int32_t* idx = f ? bl.idx[1] : bl.idx[0];
        const int u = idx[(row0 * n_qtiles + 2 * pair + k) * bl.max + c];
        if (u < 0 || u >= n_ktiles) continue;
        bool full = f == 1;
        if (!full) {
          // a partial tile the mask_mod drops whole keeps nothing; one it keeps whole
          // needs no per-element mask
          if constexpr (kDoc) {
            if (!bits_has(doc_bits(k), u)) continue;
            full = tile_class_of(k ? lo_last[1] : lo_last[0], k ? hi_first[1] : hi_first[0], u * kBN, kBN,
                                 Skv) == kTileFull;
          } else {
            if (u < sel(lo, k) || u >= sel(hi, k)) continue;
            full = tile_class<MASK>(sel(q0, k), sel(q1, k), u * kBN, kBN, mk) == kTileFull;
          }
        }
        const uint32_t bit = 1u << (u & 31);
        if (full) atomicOr(full_bits(k) + (u >> 5), bit);
        atomicOr(act_bits(k) + (u >> 5), bit);
      }
    }
  }
}

// PERSIST: one CTA per SM loops over the items blockIdx.x, blockIdx.x + gridDim.x, ...
// (analytic masks, one MMA issuer); an item is a unit or a part of one of the last units'
// key ranges (FwdParams::n_full).  The K/V ring and every barrier's phases run on across
// items, so the next item's first key/value tiles load while the current one drains; the
// producer reloads the Q tiles once the S products of the previous item have completed
// (q_free, committed by the issuer at the item's last step, before its P.V products).
// The first P.V of a tile in an item, which overwrites its O accumulator, needs no barrier
// of its own: it waits for that tile's first P of the item, which the softmax warpgroup
// writes only after its epilogue has read O of the previous item.
template <int D, typename T, int SCORE, int MASK, bool BLOCKS, bool PERSIST = false>
__global__ void __launch_bounds__(kFwdThreads, 1)
    flex_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  using L = FwdSmem<D, BLOCKS, is_doc_mask(MASK)>;
  constexpr int NS = L::kSlots;

  constexpr int kChunks = D / 64;
  constexpr uint32_t kTmemCols = 512;
  constexpr uint32_t kIdescS = idesc_f16(DtypeBits<T>::kFmt, kBM, kBN, 0);
  constexpr uint32_t kIdescPV = idesc_f16(DtypeBits<T>::kFmt, kBM, D, 1);

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
  auto bar_drain = [&](int k) { return sbase + L::kBarOff + 8u * (9 + 2 * NS + k); };
  const uint32_t bar_qfree = sbase + L::kBarOff + 8u * (11 + 2 * NS);
  uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(sgen + L::kTmemPtrOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sgen + L::kTmemPtrOff + 4);
  uint32_t* rec_smem = reinterpret_cast<uint32_t*>(sgen + L::kRecOff);  // [NS] per V slot, [NS] first

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---------------------------------------------------------------- work unit
  // Per query tile k of the pair.  Read through sel() wherever k is not a compile-time
  // constant, so that no array is indexed at run time (that would put it in local memory).
  constexpr bool kDoc = MASK == kMaskDocument || MASK == kMaskDocumentCausal;
  static_assert(!PERSIST || (!BLOCKS && !kDoc), "the persistent kernel covers the analytic masks");
  int bh, pair, h, b, bkv;
  int q0[2], q1[2], lo[2], hi[2];
  auto sel = [](const int (&a)[2], int k) { return k ? a[1] : a[0]; };
  MaskArgs mk = p.mask;
  // unit -> (b, h, pair of query tiles), later (heavier) pairs first (unit_coords)
  auto set_unit = [&](int unit) {
    unit_coords(p, unit, bh, pair);
    h = bh % p.H;
    b = bh / p.H;
    bkv = b * p.Hkv + h / p.G;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int qt = 2 * pair + k;
      q0[k] = qt * kBM;
      q1[k] = min(q0[k] + kBM, p.Sq);
      lo[k] = hi[k] = 0;
      if (qt < p.n_qtiles && !kDoc) tile_range<MASK>(q0[k], q1[k], kBN, mk, lo[k], hi[k]);
    }
  };
  // item -> (unit, part): items from n_full on take part (item - n_full) % n_parts of
  // unit n_full + (item - n_full) / n_parts, a contiguous share of each tile's key range
  // (the per-unit kernel runs item blockIdx.x, the persistent kernel a list of items)
  auto item_unit = [&](int item, int& part) {
    part = -1;
    if (item < p.n_full) return item;
    const int sidx = (item - p.n_full) / p.n_parts;
    part = item - p.n_full - sidx * p.n_parts;
    return p.n_full + sidx;
  };
  auto set_item = [&](int item) {
    int part;
    set_unit(item_unit(item, part));
    if (part >= 0) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int n = hi[k] - lo[k];
        if (n > 0) {
          const int a = lo[k] + n * part / p.n_parts;
          hi[k] = lo[k] + n * (part + 1) / p.n_parts;
          lo[k] = a;
        }
      }
    }
  };
  set_item(blockIdx.x);
  if constexpr (kDoc) {
    mk.off_q += static_cast<int64_t>(b) * (mk.n_docs + 1);
    mk.off_kv += static_cast<int64_t>(b) * (mk.n_docs + 1);
  }
  // The items of this CTA: one per round of gridDim.x items, in snake order (odd rounds
  // reversed), so that an item list sorted heaviest first spreads evenly over the CTAs;
  // items from item_end on do not exist.  The per-unit kernel has one round: blockIdx.x.
  const int item_end = PERSIST ? p.n_items : static_cast<int>(blockIdx.x) + 1;
  const int item_step = PERSIST ? static_cast<int>(gridDim.x) : 1;
  const int n_rounds = PERSIST ? (p.n_items + item_step - 1) / item_step : 1;
  auto round_item = [&](int rr) {
    const int c = (PERSIST && (rr & 1)) ? item_step - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x);
    return rr * item_step + c;
  };

  // ---------------------------------------------------------------- visit bitmaps
  // With a block mask or a document mask the key tiles a query tile visits are a set, not
  // a range (build_visit_sets).
  constexpr bool kBits = BLOCKS || kDoc;
  uint32_t* blk = reinterpret_cast<uint32_t*>(sgen + L::kBlkOff);
  auto full_bits = [&](int k) { return blk + k * kBlkWords; };
  auto act_bits = [&](int k) { return blk + (2 + k) * kBlkWords; };
  int* doc_rows = reinterpret_cast<int*>(sgen + L::kDocOff);  // doc_floor of q0/q1-1 per tile
  if constexpr (kBits) {
    const VisitLists bl{{p.blk_num[0], p.blk_num[1]}, {p.blk_idx[0], p.blk_idx[1]}, p.blk_max, p.blk_b_stride,
                        p.blk_h_stride};
    build_visit_sets<MASK, BLOCKS>(blk, doc_rows, bl, pair, b, h, q0, q1, lo, hi, mk, p.n_qtiles, p.n_ktiles, p.Skv);
  }
  // The walk over query tile k's key tiles (valid after the setup barrier); the CTA's
  // steps are the union of both walks: j = max of the two cursors.
  auto cursor = [&](int k) {
    if constexpr (kBits) return BitCursor(act_bits(k), full_bits(k), p.n_ktiles);
    else return RangeCursor(sel(lo, k), sel(hi, k));
  };
  auto has = [&](int k, int j) -> bool {  // debug tile map only
    if constexpr (kBits) return bits_has(act_bits(k), j);
    else return j >= sel(lo, k) && j < sel(hi, k);
  };

  // ---------------------------------------------------------------- setup
  // Block masks: one MMA issuer or two for this CTA (see kTwoIssuerShare), from the
  // complete visit bitmaps; the empty barriers count one arrival per issuer and use.
  volatile int* two_flag = reinterpret_cast<volatile int*>(sgen + L::kTmemPtrOff + 8);
  if constexpr (BLOCKS) __syncthreads();
  if (threadIdx.x == 0) {
    bool two = false;
    if constexpr (BLOCKS) {
      int single = 0, steps = 0;
      for (int w = 0; w < (p.n_ktiles + 31) / 32; ++w) {
        const uint32_t a = act_bits(0)[w], c = act_bits(1)[w];
        single += __popc(a ^ c);
        steps += __popc(a | c);
      }
      two = kTwoIssuerShare * single >= steps && steps > 0;
    }
    *two_flag = two ? 1 : 0;
    mbar_init(bar_q, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), two ? 2 : 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(bar_s(k), 1);
      mbar_init(bar_p(k, 0), kBM);
      mbar_init(bar_p(k, 1), kBM);
      mbar_init(bar_o(k), 1);
    }
    mbar_init(bar_drain(0), 1);
    mbar_init(bar_drain(1), 1);
    mbar_init(bar_qfree, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_ptr), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_ptr;
  const bool two_issuers = BLOCKS && *two_flag != 0;
  const bool act0 = cursor(0).cur >= 0, act1 = cursor(1).cur >= 0;
  const bool any_work = act0 || act1;

  const uint32_t q_smem0 = sbase + static_cast<uint32_t>(L::kQOff);
  auto q_smem = [&](int k) { return q_smem0 + static_cast<uint32_t>(k * L::kTileBytes); };
  auto kv_smem = [&](int s) { return sbase + static_cast<uint32_t>(L::kKVOff + s * L::kTileBytes); };

  if (warp < kSoftmaxWarp0) {
    regs_dec<kAuxRegs>();
    if (warp == kTmaWarp && lane == 0) {
      // ============================================================ TMA producer
      int r = 0;   // key/value loads issued (the ring position, across items)
      int qn = 0;  // items whose Q tiles were loaded
      bool ok = true;
      // record of the step at max(a0.cur, a1.cur) (copies: the caller's cursors stay put)
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
      // Q of the current item (set_item state) on bar_q; u_k: query tile k has work
      auto load_q = [&](bool u0, bool u1) {
        mbar_arrive_expect_tx(bar_q, (u0 ? 1 : 0) * L::kTileBytes + (u1 ? 1 : 0) * L::kTileBytes);
        for (int k = 0; k < 2; ++k) {
          if (!(k == 0 ? u0 : u1)) continue;
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(q_smem(k) + c * L::kChunkBytes, &tmQ, bar_q, c * 64, sel(q0, k), bh);
        }
      };
      if constexpr (PERSIST) {
        // The items with work form one walk: at an item's last step the record carried
        // with V is the next item's first one, flagged kRecNewItem; that item's Q loads
        // once the issuer has released the previous Q (q_free).
        int rr = -1;  // round of the current item
        auto next_work = [&]() {  // the next round's item with work (set_item state), or item_end
          while (++rr < n_rounds) {
            const int it = round_item(rr);
            if (it >= item_end) continue;
            set_item(it);
            if (cursor(0).cur >= 0 || cursor(1).cur >= 0) return it;
          }
          return item_end;
        };
        int item = next_work();
        if (item < item_end) {
          auto c0 = cursor(0), c1 = cursor(1);
          rec_smem[NS] = make_rec(c0, c1);  // published with the Q barrier
          load_q(c0.cur >= 0, c1.cur >= 0);
          qn = 1;
          while (ok) {
            const int bkv_item = bkv;
            int nxt = item_end;
            for (int j = max(c0.cur, c1.cur); j >= 0 && ok; j = max(c0.cur, c1.cur)) {  // last to first
              if (c0.cur == j) c0.advance();
              if (c1.cur == j) c1.advance();
              uint32_t next_rec = make_rec(c0, c1);
              if (next_rec == kRecEnd) {  // the item's last step: chain the next item
                nxt = next_work();
                if (nxt < item_end) next_rec = make_rec(cursor(0), cursor(1)) | kRecNewItem;
              }
              for (int which = 0; which < 2 && ok; ++which, ++r) {
                const int s = r % NS;
                const uint32_t ph = static_cast<uint32_t>(r / NS) & 1u;
                if (!mbar_wait(bar_empty(s), ph ^ 1u, p.status, kStatusFwdTimeout, kWaitTimeoutNs) ||
                    *abort_flag) {
                  *abort_flag = 1;
                  ok = false;
                  break;
                }
                if (which == 1) rec_smem[s] = next_rec;  // released by the arrive below
                mbar_arrive_expect_tx(bar_full(s), L::kTileBytes);
                const CUtensorMap* map = which == 0 ? &tmK : &tmV;
                for (int c = 0; c < kChunks; ++c)
                  tma_load_3d(kv_smem(s) + c * L::kChunkBytes, map, bar_full(s), c * 64, j * kBN, bkv_item);
              }
            }
            if (!ok || nxt >= item_end) break;
            item = nxt;  // set_item state is the next item's
            c0 = cursor(0);
            c1 = cursor(1);
            // the previous item's S products must be done with the Q tiles
            if (!mbar_wait(bar_qfree, static_cast<uint32_t>(qn - 1) & 1u, p.status, kStatusFwdTimeout,
                           kWaitTimeoutNs)) {
              *abort_flag = 1;
              break;
            }
            load_q(c0.cur >= 0, c1.cur >= 0);
            ++qn;
          }
        }
      } else {
        auto c0 = cursor(0), c1 = cursor(1);
        const bool u0 = c0.cur >= 0, u1 = c1.cur >= 0;
        if (u0 || u1) {
          // The first record is published with the Q barrier, which the issuer waits on first.
          rec_smem[NS] = make_rec(c0, c1);
          load_q(u0, u1);
          qn = 1;
          for (int j = max(c0.cur, c1.cur); j >= 0 && ok; j = max(c0.cur, c1.cur)) {  // last to first
            if (c0.cur == j) c0.advance();
            if (c1.cur == j) c1.advance();
            const uint32_t next_rec = make_rec(c0, c1);
            for (int which = 0; which < 2 && ok; ++which, ++r) {
              const int s = r % NS;
              const uint32_t ph = static_cast<uint32_t>(r / NS) & 1u;
              if (!mbar_wait(bar_empty(s), ph ^ 1u, p.status, kStatusFwdTimeout, kWaitTimeoutNs) ||
                  *abort_flag) {
                *abort_flag = 1;
                ok = false;
                break;
              }
              if (which == 1) rec_smem[s] = next_rec;  // released by the arrive below
              mbar_arrive_expect_tx(bar_full(s), L::kTileBytes);
              const CUtensorMap* map = which == 0 ? &tmK : &tmV;
              for (int c = 0; c < kChunks; ++c)
                tma_load_3d(kv_smem(s) + c * L::kChunkBytes, map, bar_full(s), c * 64, j * kBN, bkv);
            }
          }
        }
      }
      // Every load issued must land before the CTA can exit.
      const int issued = r;
      for (int e = issued - NS < 0 ? 0 : issued - NS; e < issued; ++e)
        mbar_wait(bar_full(e % NS), static_cast<uint32_t>(e / NS) & 1u, p.status, kStatusFwdTimeout,
                  kWaitTimeoutNs);
      if (qn > 0)
        mbar_wait(bar_q, static_cast<uint32_t>(qn - 1) & 1u, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
    } else if (!two_issuers && warp == kMmaWarp && lane == 0) {
      // ============================================================ MMA issuer (both tiles)
      // the first unit's Q (the persistent kernel waits for later units' in its item loop)
      bool ok = true;
      if (any_work) {
        ok = mbar_wait(bar_q, 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
        tc_fence_after();
      }
      int np[2] = {0, 0};
      // descriptor of chunk 0 / k-step 0; k-step kk adds ((kk/4)*chunk + (kk%4)*32) >> 4
      const uint64_t dq0 = smem_desc(q_smem(0), 16, 1024, kSwizzle128B);
      auto issue_s = [&](int k, int slot) {
        const uint32_t d = tmem + 128u * k;
        const uint64_t aq = dq0 + static_cast<uint64_t>((k * L::kTileBytes) >> 4);
        const uint64_t bk = smem_desc(kv_smem(slot), 16, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk / 4) * L::kChunkBytes + (kk % 4) * 32) >> 4);
          mma_ss(d, aq + off, bk + off, kIdescS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int k, int slot, bool acc, int kk0, int kk1) {
        const uint32_t d = tmem + 256u + 128u * k;
        const uint32_t a = tmem + 128u * k;
        const uint64_t bv = smem_desc(kv_smem(slot), L::kChunkBytes, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk)
          mma_ts(d, a + 8u * kk, bv + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      // s_ready[k]: S_k of the current key tile was issued during the previous step.
      bool s_ready[2] = {false, false}, started[2] = {false, false};
      // P_k V_j for query tile k (a compile-time constant, so the per-tile state stays in
      // registers), then S_k of its next key tile if that is the next step's tile (pre), or
      // the O_k completion signal after its last key tile (last); otherwise S_k waits for the
      // step of its next key tile.
      auto tile_step = [&](auto kc, bool pre, bool last, int rK, int sV, bool& next_k_ready) -> bool {
        constexpr int k = decltype(kc)::value;
        s_ready[k] = false;
        const uint32_t par = static_cast<uint32_t>(np[k]) & 1u;
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(bar_p(k, half), par, p.status, kStatusFwdTimeout, kWaitTimeoutNs)) return false;
          tc_fence_after();
          issue_pv(k, sV, started[k], 4 * half, 4 * half + 4);
        }
        started[k] = true;
        ++np[k];
        if (pre) {
          const int rK2 = rK + 2;  // K of the next step
          if (!next_k_ready) {
            if (!mbar_wait(bar_full(rK2 % NS), static_cast<uint32_t>(rK2 / NS) & 1u, p.status,
                           kStatusFwdTimeout, kWaitTimeoutNs))
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
      // One pass over the steps.  The persistent kernel's items chain their steps: the
      // record of an item's last step is followed by the first record of the next item
      // with work, flagged kRecNewItem, so the loop runs on across items.  (An item loop
      // around the step loop measured 13-18 % slower on B200 in the per-unit kernel from
      // 48 key tiles per query tile on, and 6-14 % per item in the persistent kernel.)
      bool run = any_work;
      if constexpr (PERSIST) {
        if (!any_work) {  // the CTA's first item with work is a later one: bar_q's first phase
          run = false;
          for (int rr = 1; rr < n_rounds && !run; ++rr) {
            const int it = round_item(rr);
            if (it >= item_end) continue;
            set_item(it);
            run = cursor(0).cur >= 0 || cursor(1).cur >= 0;
          }
          if (run) {
            ok = mbar_wait(bar_q, 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
            tc_fence_after();
          }
        }
      }
      if (run) {
        uint32_t rec = rec_smem[NS];  // published with the Q barrier
        [[maybe_unused]] int qn = 1;  // items started (the Q barrier's phase)
        for (int t = 0; !(rec & kRecEnd) && ok; ++t) {
          if constexpr (PERSIST) {
            if (rec & kRecNewItem) {  // the next item's Q (loaded once q_free let it)
              if (!mbar_wait(bar_q, static_cast<uint32_t>(qn) & 1u, p.status, kStatusFwdTimeout,
                             kWaitTimeoutNs)) {
                ok = false;
                break;
              }
              ++qn;
              tc_fence_after();
              s_ready[0] = s_ready[1] = started[0] = started[1] = false;
            }
          }
          const int rK = 2 * t, rV = rK + 1;
          const int sK = rK % NS, sV = rV % NS;
          const bool in0 = rec & kRecIn0, in1 = rec & kRecIn1;
          const bool need0 = in0 && !s_ready[0], need1 = in1 && !s_ready[1];
          if (need0 || need1) {
            // K_j was not needed before: wait for it here (otherwise the previous step did)
            if (!mbar_wait(bar_full(sK), static_cast<uint32_t>(rK / NS) & 1u, p.status,
                           kStatusFwdTimeout, kWaitTimeoutNs)) {
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
          if (!mbar_wait(bar_full(sV), static_cast<uint32_t>(rV / NS) & 1u, p.status,
                         kStatusFwdTimeout, kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          const uint32_t next_rec = rec_smem[sV];  // the next step's record came with V
          if constexpr (PERSIST) {
            // the item's last step: every S product of the item has been issued, so Q is
            // free once they complete; the next item's Q loads during this step's P.V
            if (next_rec & (kRecNewItem | kRecEnd)) mma_commit(bar_qfree);
          }
          bool next_k_ready = false;
          if (in0)
            ok = tile_step(std::integral_constant<int, 0>{}, rec & kRecPre0, rec & kRecLast0, rK, sV, next_k_ready);
          if (ok && in1)
            ok = tile_step(std::integral_constant<int, 1>{}, rec & kRecPre1, rec & kRecLast1, rK, sV, next_k_ready);
          if (!ok) break;
          mma_commit(bar_empty(sV));
          rec = next_rec;
        }
      }
      if (!ok) *abort_flag = 1;
      // Drain: all MMAs this thread issued have completed before TMEM is released.
      mma_commit(bar_drain(0));
      mbar_wait(bar_drain(0), 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
    } else if (two_issuers && (warp == kMmaWarp || warp == kMmaWarp1) && lane == 0 && any_work) {
      // ============================================================ MMA issuer of tile k
      // (k a compile-time constant in each of the two copies below)
      auto issuer = [&](auto kc) {
      constexpr int k = decltype(kc)::value;
      constexpr uint32_t in_bit = k ? kRecIn1 : kRecIn0, pre_bit = k ? kRecPre1 : kRecPre0;
      constexpr uint32_t last_bit = k ? kRecLast1 : kRecLast0;
      bool ok = mbar_wait(bar_q, 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
      tc_fence_after();
      // descriptor of chunk 0 / k-step 0; k-step kk adds ((kk/4)*chunk + (kk%4)*32) >> 4
      const uint64_t aq = smem_desc(q_smem(k), 16, 1024, kSwizzle128B);
      const uint32_t t_s = tmem + 128u * k, t_o = tmem + 256u + 128u * k;
      auto issue_s = [&](int slot) {
        const uint64_t bk = smem_desc(kv_smem(slot), 16, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>(((kk / 4) * L::kChunkBytes + (kk % 4) * 32) >> 4);
          mma_ss(t_s, aq + off, bk + off, kIdescS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int slot, bool acc, int kk0, int kk1) {
        const uint64_t bv = smem_desc(kv_smem(slot), L::kChunkBytes, 1024, kSwizzle128B);
#pragma unroll
        for (int kk = kk0; kk < kk1; ++kk)
          mma_ts(t_o, t_s + 8u * kk, bv + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                 (acc || kk > 0) ? 1u : 0u);
      };
      // s_ready: S_k of this step was issued during the previous one (its K already
      // waited for: k_ready); np: P.V steps done (the parity of the P barriers).
      bool s_ready = false, k_ready = false, started = false;
      int np = 0;
      uint32_t rec = rec_smem[NS];  // published with the Q barrier
      for (int t = 0; !(rec & kRecEnd) && ok; ++t) {
        const int rK = 2 * t, rV = rK + 1;
        const int sK = rK % NS, sV = rV % NS;
        const bool in = rec & in_bit;
        if (!k_ready && !mbar_wait(bar_full(sK), static_cast<uint32_t>(rK / NS) & 1u, p.status,
                                   kStatusFwdTimeout, kWaitTimeoutNs)) {
          ok = false;
          break;
        }
        k_ready = false;
        if (in) {
          tc_fence_after();
          if (!s_ready) {
            issue_s(sK);
            mma_commit(bar_s(k));
          }
          s_ready = false;
          mma_commit(bar_empty(sK));  // K_j is free once this thread's S_k(j) has run
        } else {
          mbar_arrive(bar_empty(sK));  // this tile skips the step: the slot was filled, release it
        }
        if (!mbar_wait(bar_full(sV), static_cast<uint32_t>(rV / NS) & 1u, p.status, kStatusFwdTimeout,
                       kWaitTimeoutNs)) {
          ok = false;
          break;
        }
        const uint32_t next_rec = rec_smem[sV];  // the next step's record came with V
        if (!in) {
          mbar_arrive(bar_empty(sV));
          rec = next_rec;
          continue;
        }
        const uint32_t par = static_cast<uint32_t>(np) & 1u;
        for (int half = 0; half < 2 && ok; ++half) {
          if (!mbar_wait(bar_p(k, half), par, p.status, kStatusFwdTimeout, kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(sV, started, 4 * half, 4 * half + 4);
        }
        if (!ok) break;
        started = true;
        ++np;
        if (rec & pre_bit) {
          const int rK2 = rK + 2;  // K of the next step
          if (!mbar_wait(bar_full(rK2 % NS), static_cast<uint32_t>(rK2 / NS) & 1u, p.status, kStatusFwdTimeout,
                         kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          k_ready = true;
          issue_s(rK2 % NS);
          mma_commit(bar_s(k));
          s_ready = true;
        } else if (rec & last_bit) {
          mma_commit(bar_o(k));
        }
        mma_commit(bar_empty(sV));
        rec = next_rec;
      }
      if (!ok) *abort_flag = 1;
      // Drain: all MMAs this thread issued have completed before TMEM is released.
      mma_commit(bar_drain(k));
      mbar_wait(bar_drain(k), 0, p.status, kStatusFwdTimeout, kWaitTimeoutNs);
      };
      if (warp == kMmaWarp) issuer(std::integral_constant<int, 0>{});
      else issuer(std::integral_constant<int, 1>{});
    }
  } else {
    regs_inc<kSoftmaxRegs>();
    // ============================================================ softmax warpgroups
    const int k = (warp - kSoftmaxWarp0) >> 2;  // query tile of this warpgroup
    const int wq = warp & 3;          // TMEM lane quarter
    const int row = wq * 32 + lane;   // row inside the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128u * k;
    const uint32_t tO = tmem + lane_off + 256u + 128u * k;
    bool ok = true;
    int n = 0;      // S tiles of this warpgroup so far (the S barrier's phase)
    int o_par = 0;  // O completions waited for (the O barrier's phase)
    for (int rr = 0; rr < n_rounds && ok; ++rr) {
      const int item = round_item(rr);
      if (item >= item_end) continue;
      if (PERSIST) set_item(item);
      const int q0k = sel(q0, k), q1k = sel(q1, k);
      const int qi = q0k + row;         // absolute query index
      const bool tile_valid = (2 * pair + k) < p.n_qtiles;
      const bool write_map = p.tile_map != nullptr && bh == 0 && tile_valid && threadIdx.x % 128 == 0;
      const int qt = 2 * pair + k;

      const bool act_k = cursor(k).cur >= 0;
      if (write_map) {
        for (int u = 0; u < p.n_ktiles; ++u)
          if (!act_k || !has(k, u)) p.tile_map[static_cast<int64_t>(qt) * p.n_ktiles + u] = kTileEmpty;
      }

      float m_used = -INFINITY;  // running max in log2 units (the reference of P and O)
      float l_sum = 0.f;
      const float sc = SCORE == kScoreAlibi ? 1.0f : p.scale_log2;
      float slope2 = 0.f;
      if (SCORE == kScoreAlibi)
        slope2 = (p.slopes ? __ldg(p.slopes + h) : exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(p.H))) *
                 kLog2e;
      // Document rules: this row's kept interval, looked up once (a binary search over the
      // boundaries); the tile classes come from the visit bitmaps.
      int64_t row_lo = 0, row_hi = -1;
      if constexpr (kDoc) row_interval<MASK>(qi, mk, row_lo, row_hi);

      int nu = 0;  // key tiles of this unit so far
      // Key tiles from last to first: with alibi the bias grows with the key index, so the
      // row maximum is met on the first tile and the lazy rescale of O almost never runs.
      auto cur = cursor(k);
      for (int j = cur.cur; j >= 0; j = cur.cur, ++n, ++nu) {
        // With a block mask the class comes from the walk (FULL listed or not).
        const int cls_blk =
            cur.cur_full ? (j * kBN + kBN > p.Skv ? kTileFullRagged : kTileFull) : kTilePartial;
        cur.advance();
        // Warp-uniform decision: the TMEM loads below are warp-collective.
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
        // Alibi: the bias slope2 * c of column c comes from four packed chains (columns
        // 8i + 2r, 8i + 2r + 1), each stepped by 8 * slope2; the part common to the tile,
        // slope2 * (k0 - qi), joins the running max instead of every element.  The _rn
        // operations are never fused, so every instantiation rounds them alike.
        const float base = SCORE == kScoreAlibi ? __fmul_rn(slope2, static_cast<float>(k0 - qi)) : 0.f;
        if (SCORE == kScoreAlibi) {
          const uint64_t scl2 = pack2(p.scale_log2, p.scale_log2);
          const uint64_t astep = pack2(__fmul_rn(8.f, slope2), __fmul_rn(8.f, slope2));
          uint64_t b0 = pack2(0.f, slope2), b1 = pack2(__fmul_rn(2.f, slope2), __fmul_rn(3.f, slope2));
          uint64_t b2 = pack2(__fmul_rn(4.f, slope2), __fmul_rn(5.f, slope2));
          uint64_t b3 = pack2(__fmul_rn(6.f, slope2), __fmul_rn(7.f, slope2));
  #pragma unroll
          for (int c = 0; c < kBN; c += 8) {
            unpack2(fma2(pack2(s[c], s[c + 1]), scl2, b0), s[c], s[c + 1]);
            unpack2(fma2(pack2(s[c + 2], s[c + 3]), scl2, b1), s[c + 2], s[c + 3]);
            unpack2(fma2(pack2(s[c + 4], s[c + 5]), scl2, b2), s[c + 4], s[c + 5]);
            unpack2(fma2(pack2(s[c + 6], s[c + 7]), scl2, b3), s[c + 6], s[c + 7]);
            b0 = add2(b0, astep);
            b1 = add2(b1, astep);
            b2 = add2(b2, astep);
            b3 = add2(b3, astep);
          }
        }
        if (cls != kTileFull) {
          int c_lo, c_hi;
          if (kBits && cls == kTileFullRagged)
            col_interval<kMaskNone>(qi, k0, mk, c_lo, c_hi);
          else
            if constexpr (kDoc) col_interval_of(row_lo, row_hi, k0, c_lo, c_hi);
            else col_interval<MASK>(qi, k0, mk, c_lo, c_hi);
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
        const float mx = __fadd_rn(max3f(mx0, mx1, fmaxf(mx2, mx3)) * sc, base);
        const bool need = mx > m_used + kRescaleThreshold;  // false while both are -inf
        if (__any_sync(0xffffffffu, need)) {
          float alpha = 1.0f;
          if (need) {
            alpha = ex2_approx(m_used - mx);  // 0 when m_used == -inf
            m_used = mx;
            l_sum *= alpha;
          }
          if (nu > 0) {  // the unit's first tile finds O empty
            const uint64_t a2 = pack2(alpha, alpha);
  #pragma unroll 1
            for (int c = 0; c < D; c += 32) {
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
        const float m_safe = m_used == -INFINITY ? 0.f : m_used;
        const uint64_t sc2 = pack2(sc, sc);
        const float nm = __fsub_rn(base, m_safe);
        const uint64_t nm2 = pack2(nm, nm);
        uint64_t acc2 = 0;  // two running partial sums (0.0f, 0.0f)
  #pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
  #pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = 64 * half + 2 * i;
            const uint64_t x2 = fma2(pack2(s[c], s[c + 1]), sc2, nm2);
            uint64_t e2;
            if (emu_pair(i)) {
              e2 = exp2_poly2(x2);
            } else {
              float x0, x1;
              unpack2(x2, x0, x1);
              e2 = pack2(ex2_approx(x0), ex2_approx(x1));
            }
            acc2 = add2(acc2, e2);
            float e0, e1;
            unpack2(e2, e0, e1);
            pk[i] = DtypeBits<T>::pack(e0, e1);
          }
          tmem_st32(tS + 32u * half, pk);
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar_p(k, half));
        }
        float a0, a1;
        unpack2(acc2, a0, a1);
        l_sum += a0 + a1;
      }
      if (!ok) *abort_flag = 1;

      // ---------------------------------------------------------------- epilogue
      if (tile_valid) {
        bool ran = ok && act_k;
        if (ran) {
          const bool got = mbar_wait(bar_o(k), static_cast<uint32_t>(o_par) & 1u, p.status, kStatusFwdTimeout,
                                     kWaitTimeoutNs);
          ++o_par;
          if (!__all_sync(0xffffffffu, got)) {
            *abort_flag = 1;
            ran = false;
          }
          tc_fence_after();
        }
        // The output row's address is recomputed from the item index behind an opaque copy,
        // so that the compiler keeps neither it nor the head index live through the key
        // tiles (in the persistent loop it cannot rebuild them from blockIdx).
        int opart;
        const int ou = item_unit(opaque_int(item), opart);
        int obh, opair;
        unit_coords(p, ou, obh, opair);
        const int oqi = (2 * opair + k) * kBM + row;
        const bool row_ok = oqi < p.Sq;
        // A row has mass iff it ever saw a kept (finite) score.  The polynomial 2^x returns
        // ~2^-125 rather than 0 for masked scores, so l_sum alone cannot tell.
        const bool has_mass = ran && m_used != -INFINITY && l_sum > 0.f;
        T* orow = reinterpret_cast<T*>(p.o) + (static_cast<int64_t>(obh) * p.Sq + oqi) * D;
        if (opart >= 0) {
          // A part of a split unit.  Per warp (32 rows) the parts arrive on a counter; all
          // but the last leave their rows' unnormalised O and (max, sum) in the workspace
          // and count them ready; the last waits for those (their warps are past their
          // key tiles, so the wait is their write time) and merges them with its own O,
          // still in TMEM.  No warp waits for another of its own CTA.  A part's O is
          // stored as [D / 4][kBM rows] float4s: the lanes of a warp, 32 consecutive rows,
          // write and read 512 contiguous bytes per instruction.
          const int64_t sidx = ou - p.n_full;
          const int64_t slot0 = sidx * p.n_parts * 2 + k;  // (unit, part 0, tile k)
          unsigned long long* arrived = p.part_cnt + ((sidx * 2 + k) * 4 + wq) * 2;
          unsigned long long* ready = arrived + 1;
          unsigned done = 0;
          if (lane == 0) done = tagged_add(arrived, p.part_tag);
          done = __shfl_sync(0xffffffffu, done, 0);
          const float m_own = has_mass ? m_used : -INFINITY;
          const float l_own = has_mass ? l_sum : 0.f;
          constexpr int64_t kPart4 = kBM * D / 4;  // float4s of one (part, tile) block
          if (done != static_cast<unsigned>(p.n_parts - 1)) {
            float4* dst = reinterpret_cast<float4*>(p.part_o) + (slot0 + 2 * opart) * kPart4 + row;
  #pragma unroll 1
            for (int c = 0; c < D; c += 32) {
              uint32_t r[32];
              if (ran) {
                tmem_ld32(tO + c, r);
              } else {
  #pragma unroll
                for (int e = 0; e < 32; ++e) r[e] = 0u;
              }
  #pragma unroll
              for (int v = 0; v < 8; ++v)
                dst[(c / 4 + v) * kBM] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                                     __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            }
            p.part_ml[(slot0 + 2 * opart) * kBM + row] = make_float2(m_own, l_own);
            __threadfence();  // this row's part is visible before the warp counts it ready
            __syncwarp();
            if (lane == 0) tagged_add(ready, p.part_tag);
            continue;
          }
          bool got = true;
          if (lane == 0)
            got = wait_tagged_at_least(ready, p.part_tag, static_cast<unsigned>(p.n_parts - 1), p.status,
                                       kStatusFwdTimeout, kWaitTimeoutNs);
          got = __shfl_sync(0xffffffffu, got, 0);  // (on a timeout the status says so; merged anyway)
          __threadfence();
          if (lane == 0) {  // every part is done with the counters: back to 0 under this tag (a
            const unsigned long long zero = static_cast<unsigned long long>(p.part_tag) << 32;
            *arrived = zero;  // replayed graph brings the same tag again)
            *ready = zero;
          }
          // merge: M = max of the maxima, L = sum of l_i 2^(m_i - M), O = sum of
          // O_i 2^(m_i - M) / L (parts without mass weigh 0), summed in part order with
          // this warp's own part in its place, so that the result does not depend on
          // which part arrived last
          float mi[kMaxParts], li[kMaxParts], wi[kMaxParts];
          float M = -INFINITY;
  #pragma unroll
          for (int i = 0; i < kMaxParts; ++i) {
            float2 ml = make_float2(-INFINITY, 0.f);
            if (i == opart) ml = make_float2(m_own, l_own);
            else if (i < p.n_parts) ml = __ldcg(p.part_ml + (slot0 + 2 * i) * kBM + row);
            mi[i] = ml.x;
            li[i] = ml.y;
            M = fmaxf(M, ml.x);
          }
          float L = 0.f;
  #pragma unroll
          for (int i = 0; i < kMaxParts; ++i) {
            wi[i] = mi[i] == -INFINITY ? 0.f : ex2_approx(mi[i] - M);
            L = fmaf(li[i], wi[i], L);
          }
          const bool mass = got && M != -INFINITY && L > 0.f;
          const float invL = mass ? 1.0f / L : 0.f;
  #pragma unroll
          for (int i = 0; i < kMaxParts; ++i) wi[i] *= invL;
          const float4* src = reinterpret_cast<const float4*>(p.part_o) + slot0 * kPart4 + row;
  #pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t r[32];
            if (ran) {
              tmem_ld32(tO + c, r);
            } else {
  #pragma unroll
              for (int e = 0; e < 32; ++e) r[e] = 0u;
            }
            float acc[32];
  #pragma unroll
            for (int e = 0; e < 32; ++e) acc[e] = 0.f;
  #pragma unroll 1
            for (int i = 0; i < p.n_parts; ++i) {
              const float wpart = i == 0 ? wi[0] : i == 1 ? wi[1] : i == 2 ? wi[2] : wi[3];
              float4 x[8];
              if (i == opart) {
  #pragma unroll
                for (int v = 0; v < 8; ++v)
                  x[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                     __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
              } else {
  #pragma unroll
                for (int v = 0; v < 8; ++v) x[v] = __ldcg(src + 2 * i * kPart4 + (c / 4 + v) * kBM);
              }
  #pragma unroll
              for (int v = 0; v < 8; ++v) {
                acc[4 * v] = fmaf(wpart, x[v].x, acc[4 * v]);
                acc[4 * v + 1] = fmaf(wpart, x[v].y, acc[4 * v + 1]);
                acc[4 * v + 2] = fmaf(wpart, x[v].z, acc[4 * v + 2]);
                acc[4 * v + 3] = fmaf(wpart, x[v].w, acc[4 * v + 3]);
              }
            }
            if (row_ok) {
              uint32_t w[16];
  #pragma unroll
              for (int e = 0; e < 16; ++e) w[e] = DtypeBits<T>::pack(acc[2 * e], acc[2 * e + 1]);
              uint4* od = reinterpret_cast<uint4*>(orow + c);
  #pragma unroll
              for (int v = 0; v < 4; ++v) od[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
            }
          }
          if (row_ok && p.lse != nullptr)
            p.lse[static_cast<int64_t>(obh) * p.Sq + oqi] = mass ? (M + lg2_approx(L)) * kLn2 : -INFINITY;
          continue;
        }
        const float inv = has_mass ? 1.0f / l_sum : 0.f;
  #pragma unroll 1
        for (int c = 0; c < D; c += 32) {
          uint32_t r[32];
          // defined on both paths: an undefined r would stay live around the item loop
          if (ran) {
            tmem_ld32(tO + c, r);
          } else {
  #pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0u;
          }
          uint32_t w[16];
  #pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = has_mass ? __uint_as_float(r[2 * e]) * inv : 0.f;
            const float bb = has_mass ? __uint_as_float(r[2 * e + 1]) * inv : 0.f;
            w[e] = DtypeBits<T>::pack(a, bb);
          }
          if (row_ok) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
  #pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
        if (row_ok && p.lse != nullptr) {
          p.lse[static_cast<int64_t>(obh) * p.Sq + oqi] =
              has_mass ? (m_used + lg2_approx(l_sum)) * kLn2 : -INFINITY;
        }
      }
    }  // item
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace flexattn
