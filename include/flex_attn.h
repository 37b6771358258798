/*
 * flex_attn.h -- C ABI of the B200 (sm_100a) flex-attention library.
 *
 * The library computes the fused attention forward pass
 *
 *     O = softmax( mask_mod( score_mod( scale * Q K^T ) ) ) V,   LSE = log-sum-exp per row
 *
 * with PyTorch flex_attention's per-element hooks, and a decode variant for one
 * query row against a KV cache of dynamic length.
 *
 * Sources for the operation (page title, section):
 *  - FlyDSL PR 931 "Add flex_attention (score_mod / mask_mod) on the generic
 *    flash-attention kernel", Summary: score_mod(score, b, h, q_idx, kv_idx) gets the
 *    already scaled score and runs before the mask; mask_mod(b, h, q_idx, kv_idx)
 *    keeps or drops an element; built-in alibi / sliding_window / causal mods;
 *    fully masked rows give O = 0 and LSE = -inf.
 *  - torch-mlir PR 4366 "[TORCH] Added flex_attention hop function", Description:
 *    the operands query, key, value, scale, enable_gqa, return_lse.
 *  - IREE issue 19015 "[ROCM] Support dynamic key-value cache sequence length",
 *    example IR: decode with q [B,H,1,D], K/V cache [B,H,?,D], an f16 additive mask
 *    [B,H,1,?] and an f32 accumulation region.
 *
 * Conventions shared by every entry point
 *  - Pointers named q/k/v/o/lse/kv_len/mask/workspace are DEVICE pointers on the
 *    current CUDA device, owned by the caller.  The library keeps no per-call state
 *    and allocates no device memory.
 *  - Layouts are dense row-major: Q/O [B, H, Sq, D]; K/V [B, Hkv, Skv, D];
 *    LSE [B, H, Sq] fp32 (natural log); KV cache [B, Hkv, cap, D].
 *  - Every pointer must be 16-byte aligned.
 *  - GQA: query head h reads key/value head h / (H / Hkv); H % Hkv must be 0.
 *  - Argument checks run on the host before any launch; a failed check returns an
 *    error code and launches nothing.  Work is enqueued on `stream` and the call
 *    returns without synchronising.
 *  - Problems that only the device can see (a kv_len outside [0, cap], a wait that
 *    ran out of time) set bits in a device status word instead of trapping.  Each call
 *    can name its own word (status_out in flex_mod_params_t / flex_decode_params_t:
 *    a caller-owned device uint32, OR-ed into, never cleared by the library), so that
 *    calls on different streams can tell whose problem a bit is and read it with a
 *    stream-ordered copy.  Calls that name none report into one word per device that
 *    all such calls share; flex_attn_device_status() reads it (and synchronises the
 *    device to do so).  The bits are listed with flex_attn_device_status().
 */
#ifndef FLEX_ATTN_H_
#define FLEX_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* flex_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
  FLEX_OK = 0,
  FLEX_ERR_INVALID_ARG = 1,   /* null pointer, bad size, H % Hkv != 0, bad mod parameter */
  FLEX_ERR_UNSUPPORTED = 2,   /* head dim or dtype the kernels do not cover */
  FLEX_ERR_MISALIGNED = 3,    /* a pointer that is not 16-byte aligned */
  FLEX_ERR_WORKSPACE = 4,     /* decode workspace missing or too small */
  FLEX_ERR_CUDA = 5,          /* a CUDA runtime/driver call failed (launch, tensor map) */
  FLEX_ERR_DEVICE_TIMEOUT = 6 /* reported through flex_attn_device_status() only */
} flex_status_t;

typedef enum { FLEX_DTYPE_BF16 = 0, FLEX_DTYPE_F16 = 1 } flex_dtype_t;

/* score_mod: applied to s = scale * q.k before any mask (FlyDSL PR 931, Summary). */
typedef enum {
  FLEX_SCORE_NONE = 0,
  FLEX_SCORE_ALIBI = 1,       /* s += slope_h * (kv_idx - q_idx), slope_h = 2^(-8 (h+1) / H) */
  FLEX_SCORE_ALIBI_SLOPES = 2 /* tensor-capturing: slope_h = mod_params->alibi_slopes[h] */
} flex_score_mod_t;

/* mask_mod: keep (q_idx, kv_idx) iff the rule holds; indices are absolute (top-left). */
typedef enum {
  FLEX_MASK_NONE = 0,
  FLEX_MASK_CAUSAL = 1,                /* causal_via_mask: kv_idx <= q_idx                  */
  FLEX_MASK_SLIDING_WINDOW = 2,        /* kv_idx <= q_idx && q_idx - kv_idx < window        */
  FLEX_MASK_KV_LE_Q_PLUS_OFFSET = 3,   /* kv_idx <= q_idx + offset (offset may be negative) */
  FLEX_MASK_CAUSAL_FAST = 4,           /* causal=True: the same keep rule as CAUSAL          */
  /* Tensor-capturing mask_mods (FlyDSL PR 931, Out of scope: a later phase, not defined
   * there).  Packed sequences: per batch b, mod_params->doc_offsets_q[b][0 .. n_docs]
   * are the document boundaries of the query positions and doc_offsets_kv those of the
   * keys; position p is in document d iff off[d] <= p < off[d+1] (in none otherwise).
   * Boundaries must be non-decreasing; other values cannot make a kernel read out of
   * bounds, but then the keys kept are unspecified.  The forward kernels skip exactly the
   * key tiles no row keeps; Skv at most 2048 * 128 (FLEX_ERR_UNSUPPORTED beyond). */
  FLEX_MASK_DOCUMENT = 5,              /* q_idx and kv_idx in the same document            */
  FLEX_MASK_DOCUMENT_CAUSAL = 6        /* ... and kv_idx <= q_idx                           */
} flex_mask_mod_t;

/* Tile classification written by the debug tile map (one byte per tile). */
enum { FLEX_TILE_EMPTY = 0, FLEX_TILE_FULL = 1, FLEX_TILE_PARTIAL = 2 };

#define FLEX_FLAG_TILE_MAP 1u /* write tile_map_out (see flex_mod_params_t) */

typedef struct {
  int32_t window;  /* FLEX_MASK_SLIDING_WINDOW: number of keys kept, >= 1 */
  int32_t offset;  /* FLEX_MASK_KV_LE_Q_PLUS_OFFSET */
  uint32_t flags;  /* FLEX_FLAG_* */
  /* Debug: device buffer of ceil(Sq/BM) * ceil(Skv/BN) bytes.  With FLEX_FLAG_TILE_MAP
   * set, the work units of batch 0 / head 0 write the class of every (q-tile, kv-tile)
   * they process (FULL or PARTIAL) and EMPTY for every tile they skip. */
  uint8_t* tile_map_out;
  /* Captured tensors (device memory, 4-byte aligned, owned by the caller):
   * FLEX_SCORE_ALIBI_SLOPES: alibi_slopes[H] fp32.
   * FLEX_MASK_DOCUMENT*: doc_offsets_q [B, n_docs + 1] int32 and doc_offsets_kv of the
   * same shape (NULL = the same boundaries as the queries); n_docs >= 0. */
  const float* alibi_slopes;
  const int32_t* doc_offsets_q;
  const int32_t* doc_offsets_kv;
  int32_t n_docs;
  /* Per-call device status word (device memory, 4-byte aligned, owned by the caller):
   * the kernels of this call OR their status bits into it.  NULL = the shared per-device
   * word read by flex_attn_device_status(). */
  uint32_t* status_out;
} flex_mod_params_t;

/*
 * flex_attn_fwd -- fused forward pass (FlyDSL PR 931, Summary; torch-mlir PR 4366,
 * Description).
 *
 *   q   [B, H,   Sq,  D]  dtype         k, v [B, Hkv, Skv, D]  dtype
 *   o   [B, H,   Sq,  D]  dtype (out)   lse  [B, H, Sq] fp32 (out; NULL = return_lse false)
 *   scale: multiplies q.k before score_mod; finite and > 0.
 *   score_mod_id: flex_score_mod_t; mask_mod_id: flex_mask_mod_t.
 *   mod_params: may be NULL when no mask parameter is needed.
 *   D in {64, 128}; dtype in {BF16, F16}; B, H, Hkv, Sq, Skv >= 1.
 * Accumulation is fp32; P and O are rounded to dtype with round-to-nearest-even.
 * Rows whose every key is masked get O = +0 and LSE = -inf.
 * Returns FLEX_OK or an error code (nothing is launched on error).
 */
flex_status_t flex_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                            int B, int H, int Hkv, int Sq, int Skv, int D, float scale,
                            int score_mod_id, int mask_mod_id, const flex_mod_params_t* mod_params,
                            flex_dtype_t dtype, flex_stream_t stream);

/*
 * flex_block_mask_t -- a block mask (BlockMask): per query tile of 128 rows, lists of key
 * blocks of 128 keys.  FlyDSL PR 931 (Out of scope) names block sparsity as the next
 * phase without defining it; the lists follow PyTorch's BlockMask convention:
 *   - a key block on the query tile's full list is kept whole (only kv_idx < Skv applies);
 *   - a key block on its partial list keeps the elements mask_mod keeps;
 *   - every other key block is dropped; a block on both lists counts as full.
 * Arrays are DEVICE int32, dense row-major, owned by the caller, 4-byte aligned:
 *   kv_num_blocks, full_kv_num_blocks  [batch, heads, ceil(Sq/128)]
 *   kv_indices, full_kv_indices        [batch, heads, ceil(Sq/128), max_blocks]
 * Either (num, indices) pair may be NULL (no blocks of that kind), not both.  batch is 1
 * (one mask for every batch) or B; heads is 1 or H.  Only the first num entries of an
 * index row are read; num is clamped to [0, max_blocks] on the device, an index outside
 * [0, ceil(Skv/128)) names no block, and a repeated index counts once, so no value in
 * these arrays can make the kernel read out of bounds.  The order of the entries does
 * not matter.
 */
typedef struct {
  const int32_t* kv_num_blocks;
  const int32_t* kv_indices;
  const int32_t* full_kv_num_blocks;
  const int32_t* full_kv_indices;
  int32_t max_blocks;     /* >= 1 */
  int32_t batch;          /* 1 or B */
  int32_t heads;          /* 1 or H */
  int32_t q_block_size;   /* must be 128 (FLEX_ERR_UNSUPPORTED otherwise) */
  int32_t kv_block_size;  /* must be 128 (FLEX_ERR_UNSUPPORTED otherwise) */
} flex_block_mask_t;

/*
 * flex_attn_fwd_block_sparse -- flex_attn_fwd with a block mask: the key tiles each query
 * tile visits come from block_mask instead of from the range mask_mod implies; partial
 * blocks still apply mask_mod element by element (and blocks that mask_mod drops whole are
 * skipped), full blocks apply only kv_idx < Skv.  Arguments, layouts and errors are those
 * of flex_attn_fwd, plus: block_mask non-NULL and valid as described above; Skv at most
 * 2048 * 128 = 262144 (FLEX_ERR_UNSUPPORTED beyond); mod_params->tile_map_out, if asked
 * for, records what the kernel visited (FULL, or PARTIAL for tiles it masks).
 */
flex_status_t flex_attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse,
                                         int B, int H, int Hkv, int Sq, int Skv, int D, float scale,
                                         int score_mod_id, int mask_mod_id,
                                         const flex_mod_params_t* mod_params,
                                         const flex_block_mask_t* block_mask, flex_dtype_t dtype,
                                         flex_stream_t stream);

/*
 * flex_attn_fwd_host_workspace_size -- bytes of device workspace flex_attn_fwd_host needs:
 * three chunk buffers (Q, K, V, O, LSE of one chunk of kv heads) and a table of H slopes;
 * 0 for invalid sizes.
 */
size_t flex_attn_fwd_host_workspace_size(int B, int H, int Hkv, int Sq, int Skv, int D);

/*
 * flex_attn_fwd_host -- flex_attn_fwd on HOST buffers (the forward of FlyDSL PR 931,
 * Summary, with the operands of torch-mlir PR 4366, Description, living in host memory):
 * q, k, v are read from and o, lse written to host memory in the layouts of flex_attn_fwd.
 * The work is split into about 16 chunks (ranges of kv heads of one batch, or, with 16 or
 * more batches, runs of whole batches); chunk c's
 * copy to the device, the forward on chunk c - 1 and the copy of chunk c - 2's O and LSE
 * back run at the same time (copies on two streams of the library's own, the forward on
 * `stream`), so the call takes about as long as its host-to-device copies.  The results
 * equal flex_attn_fwd's on the same values up to the summation order of key-range parts
 * (the split of a last round of units depends on the number of units per launch).
 *   q, k, v, o, lse: host pointers (lse may be NULL).  Page-locked (pinned) memory lets the
 *   copies run asynchronously and overlap; pageable memory works but serialises them.
 *   The host buffers must stay valid and untouched until `stream` has passed this call.
 *   score_mod_id, mask_mod_id, mod_params: as flex_attn_fwd; captured tensors
 *   (alibi_slopes, doc_offsets_*) are DEVICE pointers as there; FLEX_FLAG_TILE_MAP is
 *   rejected (FLEX_ERR_INVALID_ARG).
 *   workspace: device memory, at least flex_attn_fwd_host_workspace_size(...) bytes,
 *   16-byte aligned; in use until `stream` has passed this call.
 * Asynchronous on `stream`: work queued on it before the call runs first, and work queued
 * after it starts only once every copy has finished.  Calls from several host threads are
 * serialised while they enqueue (they share the library's copy streams).
 */
flex_status_t flex_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                 int Hkv, int Sq, int Skv, int D, float scale, int score_mod_id, int mask_mod_id,
                                 const flex_mod_params_t* mod_params, flex_dtype_t dtype, void* workspace,
                                 size_t workspace_bytes, flex_stream_t stream);

/*
 * flex_attn_fwd_fp8_workspace_size -- bytes of device workspace flex_attn_fwd_fp8 needs
 * (a transposed copy of V, keys padded to a multiple of 128); 0 for D other than 64, 128.
 */
size_t flex_attn_fwd_fp8_workspace_size(int B, int Hkv, int Skv, int D);

/*
 * flex_attn_fwd_fp8 -- the forward pass with 8-bit inputs (FlyDSL PR 931, Out of scope:
 * "fp8 flex paths" as a later phase).  q8, k8, v8 hold e4m3 codes (OCP E4M3FN, one byte
 * each) in the layouts of flex_attn_fwd; the values are descale_q * q8, descale_k * k8,
 * descale_v * v8.  Computes O = softmax(mask_mod(score_mod(scale * q . k))) v with
 * fp32 accumulation; the probabilities enter the P.V product rounded to e4m3 (scaled
 * into the format's range and back, see the kernel header); O is written in bf16
 * [B, H, Sq, D], LSE (natural log) in fp32 [B, H, Sq] (NULL allowed).
 *   D must be 64 or 128 (FLEX_ERR_UNSUPPORTED otherwise); scale and the descales finite, > 0.
 *   score_mod_id, mask_mod_id, mod_params: as for flex_attn_fwd (every mod, the captured
 *   tensors, the debug tile map).
 *   workspace: at least flex_attn_fwd_fp8_workspace_size(B, Hkv, Skv, D) bytes,
 *   16-byte aligned; overwritten.
 */
flex_status_t flex_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse,
                                int B, int H, int Hkv, int Sq, int Skv, int D, float scale,
                                float descale_q, float descale_k, float descale_v, int score_mod_id,
                                int mask_mod_id, const flex_mod_params_t* mod_params, void* workspace,
                                size_t workspace_bytes, flex_stream_t stream);

/*
 * flex_attn_fwd_fp8_block_sparse -- flex_attn_fwd_fp8 with a block mask: the key tiles each
 * query tile visits come from block_mask (the rules and limits of
 * flex_attn_fwd_block_sparse), the rest as flex_attn_fwd_fp8.
 */
flex_status_t flex_attn_fwd_fp8_block_sparse(const void* q8, const void* k8, const void* v8, void* o,
                                             float* lse, int B, int H, int Hkv, int Sq, int Skv, int D,
                                             float scale, float descale_q, float descale_k,
                                             float descale_v, int score_mod_id, int mask_mod_id,
                                             const flex_mod_params_t* mod_params,
                                             const flex_block_mask_t* block_mask, void* workspace,
                                             size_t workspace_bytes, flex_stream_t stream);

/*
 * flex_attn_bwd_workspace_size -- bytes of device workspace flex_attn_bwd needs
 * (per query row: -LSE in base 2 and -delta with delta = dO . O, rows padded to a multiple
 * of 128).  The contents are private to one call.
 */
size_t flex_attn_bwd_workspace_size(int B, int H, int Sq);

/*
 * flex_attn_bwd -- gradients of sum(dout * O) for the forward with the same arguments
 * (the backward pass, FlyDSL PR 931, Out of scope: a later phase; xformers 1094 "Tiny
 * upstream pr" reports dq/dk/dv mean errors of a backward).  With P the forward's
 * probabilities (recomputed from q, k and the forward's lse), delta_i = dout_i . o_i and
 * dS = P * (dout V^T - delta):  dq = scale dS K,  dk = scale dS^T Q,  dv = P^T dout, where
 * dk and dv sum over the H / Hkv query heads that share a key/value head.
 *   q, o, dout, dq [B, H, Sq, D] dtype;  k, v, dk, dv [B, Hkv, Skv, D] dtype;
 *   lse [B, H, Sq] fp32: the forward's LSE (natural log; -inf for rows without keys).
 *   scale, score_mod_id, mask_mod_id, mod_params: those of the forward (any mod
 *   flex_attn_fwd takes; with a block mask see flex_attn_bwd_block_sparse).
 *   workspace: at least flex_attn_bwd_workspace_size(B, H, Sq) bytes, 16-byte aligned.
 * Accumulation is fp32; P and dS enter the matmuls rounded to dtype (round-to-nearest-
 * even).  Rows without keys give no gradient.  Deterministic: no atomics.
 */
flex_status_t flex_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, int B, int H, int Hkv,
                            int Sq, int Skv, int D, float scale, int score_mod_id, int mask_mod_id,
                            const flex_mod_params_t* mod_params, flex_dtype_t dtype, void* workspace,
                            size_t workspace_bytes, flex_stream_t stream);

/*
 * flex_decode_params_t -- optional settings of one decode call (NULL = all defaults).
 *   split_size: cache positions per split of the split-KV decode: 0 = the library's
 *     choice (128 when H == Hkv, else 256), else 128 or 256 (FLEX_ERR_INVALID_ARG
 *     otherwise).  The result does not
 *     depend on it beyond rounding (the combine is exact in real arithmetic); smaller
 *     splits give more parallel work for short sequences and need more workspace.
 *   status_out: per-call device status word, as in flex_mod_params_t (NULL = the shared
 *     per-device word).
 */
typedef struct {
  int32_t split_size;
  uint32_t* status_out;
} flex_decode_params_t;

/*
 * flex_attn_bwd_block_sparse_workspace_size -- bytes of device workspace
 * flex_attn_bwd_block_sparse needs: flex_attn_bwd's per-row statistics plus the block
 * mask transposed to key tiles (per batch, kv head and key tile, two bitmaps over the
 * (query head of the group, query tile) pairs).  0 for invalid sizes.
 */
size_t flex_attn_bwd_block_sparse_workspace_size(int B, int H, int Hkv, int Sq, int Skv);

/*
 * flex_attn_bwd_block_sparse -- gradients of the block-sparse forward
 * (flex_attn_fwd_block_sparse) with the same arguments: flex_attn_bwd with the keep rule
 * of the block mask (block sparsity and the backward are both named as later phases on
 * FlyDSL PR 931, Out of scope).  A key block on a query tile's full list keeps every key
 * below Skv, one on its partial list the keys mask_mod keeps; every other key is dropped
 * and takes no gradient.  Arguments, layouts and errors are those of flex_attn_bwd and of
 * flex_attn_fwd_block_sparse (the block_mask rules and limits), plus:
 *   workspace: at least flex_attn_bwd_block_sparse_workspace_size(B, H, Hkv, Sq, Skv)
 *   bytes, 16-byte aligned; overwritten.
 * Deterministic: the transposed bitmaps are built with atomic ORs, whose result does
 * not depend on their order; the gradients use no atomics.
 */
flex_status_t flex_attn_bwd_block_sparse(const void* q, const void* k, const void* v, const void* o,
                                         const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                         int B, int H, int Hkv, int Sq, int Skv, int D, float scale,
                                         int score_mod_id, int mask_mod_id,
                                         const flex_mod_params_t* mod_params,
                                         const flex_block_mask_t* block_mask, flex_dtype_t dtype,
                                         void* workspace, size_t workspace_bytes, flex_stream_t stream);

/*
 * flex_attn_decode_workspace_size -- bytes of device workspace flex_attn_decode needs
 * for these sizes (the split-KV partial outputs and their log-sum-exps), whatever split
 * size the call uses (it is the size for the smallest split, 128 positions).
 */
size_t flex_attn_decode_workspace_size(int B, int H, int Hkv, int cap, int D);

/*
 * flex_attn_decode -- one query row per (batch, head) against a KV cache of
 * per-sequence dynamic length (IREE issue 19015, example IR).
 *
 *   q        [B, H, 1, D]     dtype          k_cache, v_cache [B, Hkv, cap, D] dtype
 *   kv_len   [B] int32 (device): valid length of each sequence, 0 <= kv_len[b] <= cap;
 *            positions >= kv_len[b] are never read.  kv_len[b] == 0 gives O = 0, LSE = -inf.
 *            A value outside [0, cap] sets a device status bit and that sequence's
 *            rows are written as O = 0, LSE = -inf.
 *   additive_mask [B, H, 1, cap] dtype, or NULL: added to scale * q.k (after scaling);
 *            -inf drops a position.
 *   o        [B, H, 1, D] dtype (out);  lse [B, H, 1] fp32 (out, NULL allowed).
 *   workspace: device buffer of at least flex_attn_decode_workspace_size() bytes,
 *            16-byte aligned; its contents on entry do not matter.  (A smaller buffer
 *            is accepted when it holds the partials of the split size actually used:
 *            B * H * ceil(cap / split) * (D + 1) * 4 bytes, the first part rounded up
 *            to 256 bytes.)
 *   scale: finite and > 0.  D in {64, 128}; dtype in {BF16, F16}.
 *   params: NULL or the split size and per-call status word (flex_decode_params_t).
 */
flex_status_t flex_attn_decode(const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* kv_len, const void* additive_mask, void* o,
                               float* lse, int B, int H, int Hkv, int cap, int D, float scale,
                               flex_dtype_t dtype, void* workspace, size_t workspace_bytes,
                               const flex_decode_params_t* params, flex_stream_t stream);

/*
 * flex_attn_decode_noalloc -- flex_attn_decode without a caller-supplied workspace.
 * (No counterpart on the source pages: this entry point exists for callers of this
 * library.)  Some callers cannot allocate device memory at call time: hosts that load
 * operators through a fixed interface which passes only inputs and outputs, processes
 * that reserved their whole memory budget up front, and latency-bound decode loops that
 * must not pay for cudaMalloc/cudaFree (both synchronise the device).  This variant
 * needs no workspace: it uses a scratch array of FLEX_DECODE_STATIC_SCRATCH_BYTES
 * compiled into the library, which every GPU that loads the library keeps until the
 * process exits.  It calls no allocator of any kind.
 *   Arguments, layouts and errors are those of flex_attn_decode.  This variant splits
 *   the cache into 256-position splits unless params->split_size asks for 128; sizes
 *   whose partials at that split size (B * H * ceil(cap / split) * (D + 1) * 4 bytes)
 *   exceed FLEX_DECODE_STATIC_SCRATCH_BYTES return FLEX_ERR_WORKSPACE and launch nothing.
 *   The first call on a device (and the first after that device's context was destroyed
 *   and created again) looks up the device address of the scratch array
 *   (cudaGetSymbolAddress, with that device current); make that first call before any
 *   stream capture on the device.
 *   All calls on a device share the one array and it keeps the last call's contents;
 *   the kernels write every scratch entry they read, so nothing needs clearing, but
 *   calls that overlap on the GPU (e.g. on two streams at once) race on it and must be
 *   serialised by the caller.
 */
#define FLEX_DECODE_STATIC_SCRATCH_BYTES (16u * 1024u * 1024u)
flex_status_t flex_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* kv_len, const void* additive_mask, void* o,
                                       float* lse, int B, int H, int Hkv, int cap, int D, float scale,
                                       flex_dtype_t dtype, const flex_decode_params_t* params,
                                       flex_stream_t stream);

/*
 * flex_attn_mask_eval -- debug: evaluates the device mask rule the forward kernel uses
 * into keep[Sq * Skv] (uint8, device, 1 = kept) for element-exact comparison.
 * Covers mask_mod and the j < Skv pad rule; the document rules read the boundaries of
 * batch 0 (the first n_docs + 1 entries of doc_offsets_q / doc_offsets_kv).
 */
flex_status_t flex_attn_mask_eval(int mask_mod_id, const flex_mod_params_t* mod_params,
                                  int Sq, int Skv, uint8_t* keep, flex_stream_t stream);

/*
 * flex_attn_selftest_wait_timeout -- failure-detection self-test (no counterpart on the
 * source pages).  Launches one thread that waits, with the same bounded mbarrier wait the
 * forward kernel uses, on a barrier nothing ever arrives on; after timeout_us
 * microseconds (1 .. 2,000,000) the wait gives up and sets status bit 8.  Shows that an
 * expired wait ends the kernel normally, reports through the status word, and leaves the
 * context usable.  Asynchronous on `stream`.
 */
flex_status_t flex_attn_selftest_wait_timeout(uint32_t timeout_us, flex_stream_t stream);

/* flex_attn_tile_sizes -- the (BM, BN) tile geometry the forward kernel uses for D. */
void flex_attn_tile_sizes(int D, int* bm, int* bn);

/*
 * flex_attn_device_status -- reads (and, if reset != 0, clears) the shared status word
 * of the current device: the bits of every call that named no status_out of its own,
 * whichever stream it ran on.  Synchronises the device.  (A per-call status_out holds
 * the same bits for that call alone.)  Bits:
 *   1 = a decode kv_len outside [0, cap];  2 = a forward-kernel wait ran out of time;
 *   4 = a decode-kernel wait ran out of time;  8 = the self-test wait ran out (expected);
 *   16 = a backward-kernel wait ran out of time.
 */
flex_status_t flex_attn_device_status(uint32_t* status_out, int reset);

/* flex_status_string -- a static description of a status code. */
const char* flex_status_string(flex_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* FLEX_ATTN_H_ */
