// flex_attn_api.cu -- the C ABI declared in include/flex_attn.h: host-side argument
// checks, TMA tensor-map encoding and the choice of launcher (head dim, block mask);
// the launchers in flex_fwd_d*.cu and flex_decode_launch.cu dispatch over (dtype,
// score_mod, mask_mod) and launch on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "flex_attn.h"
#include "launch.cuh"
#include "mask_rules.cuh"

namespace flexattn {

// Device status word (bits documented with flex_attn_device_status).
__device__ unsigned int g_status;

namespace {

// Largest key-tile count per query tile that runs on the persistent forward kernel.
constexpr int64_t kPersistMaxKeyTiles = 32;
// Largest K + V footprint (bytes) with which causal-like masks run persistent.
constexpr int64_t kPersistRisingMaxKvBytes = int64_t{80} << 20;


bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// ---------------------------------------------------------------- tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [rows3 x rows x D] 16-bit tensor, box = 64 elements x box_rows rows x 1, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, flex_dtype_t dt, int D, int rows, int64_t outer,
              int box_rows = kBM) {
  auto fn = encode_fn();
  if (!fn) return false;
  const CUtensorMapDataType t = dt == FLEX_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(D) * 2 * rows};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, t, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The decode's additive mask [B, H, 1, cap] as a [cap, H, B] 16-bit tensor, box = 64
// positions x `rows` heads x 1, no swizzle (cap must be a multiple of 8: 16-byte strides).
bool make_map_mask(CUtensorMap* map, const void* base, flex_dtype_t dt, int cap, int H, int B, int rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const CUtensorMapDataType t = dt == FLEX_DTYPE_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cap), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(cap) * 2, static_cast<cuuint64_t>(cap) * 2 * H};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(kDtKeys), static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, t, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [outer x rows x inner] bytes, box = 128 bytes x 128 rows x 1, 128-byte swizzle (the
// 8-bit forward's tiles; inner must be a multiple of 16; a box past inner or rows reads
// zeros, which pads 64-byte rows and 64-row V^T tiles to the 128-byte tile width).
bool make_map_u8(CUtensorMap* map, const void* base, int64_t inner, int64_t rows, int64_t outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(inner * rows)};
  cuuint32_t box[3] = {128, static_cast<cuuint32_t>(kBM), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Scratch for flex_attn_decode_noalloc: compiled into the library so that callers who
// cannot allocate device memory still get a workspace.  One copy per device, shared by
// every call on that device.
__device__ __align__(256) unsigned char g_decode_scratch[FLEX_DECODE_STATIC_SCRATCH_BYTES];

// Id of the context current on this thread (driver entry points, so the runtime does not
// create a context just to answer), or false when none is current.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(a);
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(b);
    }
  });
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device addresses of the library's __device__ symbols (host code sees only host-side
// stand-ins under those names).  Looked up once per device and context: a context that
// was destroyed and created again (cudaDeviceReset) loads the module anew, at a new
// address, so the cache is keyed on the context's id.
enum Symbol { kSymStatus = 0, kSymScratch = 1 };

void* symbol_ptr(Symbol which) {
  constexpr int kMaxDevices = 64;
  struct Entry {
    unsigned long long ctx;
    void* addr[2];
  };
  static Entry cache[kMaxDevices] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  if (have_id) {
    std::lock_guard<std::mutex> g(mu);
    if (cache[dev].ctx == id && cache[dev].addr[which]) return cache[dev].addr[which];
  }
  void* p = nullptr;
  const cudaError_t e = which == kSymStatus ? cudaGetSymbolAddress(&p, g_status)
                                            : cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) return nullptr;
  if (!have_id) have_id = current_context_id(&id);  // the lookup made the context current
  if (have_id) {
    std::lock_guard<std::mutex> g(mu);
    if (cache[dev].ctx != id) cache[dev] = Entry{id, {nullptr, nullptr}};
    cache[dev].addr[which] = p;
  }
  return p;
}

void* decode_scratch_ptr() { return symbol_ptr(kSymScratch); }

// Workspace of the forward's split units, one per (context, stream) and kept for the
// process's life: calls on one stream run in order and share it, calls on different
// streams never do.  Sized for the most a launch can use (R * parts <= SMs split rows of
// both tiles at D = 128); created zeroed on first use.  Each call takes the next tag for
// the tagged counters, so they are never reset between calls.
struct SplitWorkspace {
  void* base;
  unsigned tag;
};

bool split_workspace(cudaStream_t stream, int sms, SplitWorkspace* out, size_t* cnt_bytes_out,
                     size_t* ml_bytes_out) {
  struct Entry {
    unsigned long long ctx;
    cudaStream_t stream;
    void* base;
    unsigned tag;
  };
  static std::vector<Entry> entries;
  static std::mutex mu;
  unsigned long long id = 0;
  if (!current_context_id(&id)) return false;
  const size_t rows = static_cast<size_t>(sms) * 2 * kBM;
  const size_t cnt_bytes = (static_cast<size_t>(sms) * 2 * 4 * 2 * sizeof(unsigned long long) + 255) / 256 * 256;
  const size_t ml_bytes = rows * sizeof(float2);
  const size_t bytes = cnt_bytes + ml_bytes + rows * 128 * sizeof(float);
  std::lock_guard<std::mutex> lock(mu);
  for (Entry& e : entries) {
    if (e.ctx == id && e.stream == stream) {
      out->base = e.base;
      out->tag = ++e.tag == 0 ? ++e.tag : e.tag;  // tag 0 is the zeroed state
      *cnt_bytes_out = cnt_bytes;
      *ml_bytes_out = ml_bytes;
      return true;
    }
  }
  void* base = nullptr;
  if (cudaMalloc(&base, bytes) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (cudaMemsetAsync(base, 0, cnt_bytes, stream) != cudaSuccess) {  // ordered before the launch
    cudaFree(base);
    return false;
  }
  entries.push_back({id, stream, base, 1u});
  out->base = base;
  out->tag = 1u;
  *cnt_bytes_out = cnt_bytes;
  *ml_bytes_out = ml_bytes;
  return true;
}

// Streaming multiprocessors of the current device (looked up once per device).
int sm_count() {
  constexpr int kMaxDevices = 64;
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  int n = cache[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

// The status word a call's kernels report into: the caller's own, or the shared one.
unsigned* status_for(uint32_t* status_out) {
  if (status_out) return reinterpret_cast<unsigned*>(status_out);
  return static_cast<unsigned*>(symbol_ptr(kSymStatus));
}

// ---------------------------------------------------------------- mask evaluation (debug)

// Composes exactly the decisions the forward kernel takes for element (i, j): is the key
// tile of j visited by the query tile of i, and if so FULL or inside the row interval.
template <int MASK>
__global__ void mask_eval_kernel(MaskArgs m, int Sq, int Skv, uint8_t* keep) {
  const int64_t total = static_cast<int64_t>(Sq) * Skv;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(idx / Skv), j = static_cast<int>(idx % Skv);
    const int q0 = (i / kBM) * kBM, q1 = min(q0 + kBM, Sq);
    int t_lo, t_hi;
    tile_range<MASK>(q0, q1, kBN, m, t_lo, t_hi);
    const int u = j / kBN, k0 = u * kBN;
    uint8_t kv = 0;
    if (u >= t_lo && u < t_hi) {
      if (tile_class<MASK>(q0, q1, k0, kBN, m) == kTileFull) {
        kv = 1;
      } else {
        int lo, hi;
        col_interval<MASK>(i, k0, m, lo, hi);
        kv = (j - k0 >= lo && j - k0 <= hi) ? 1 : 0;
      }
    }
    keep[idx] = kv;
  }
}

int decode_splits(int cap, int split) { return (cap + split - 1) / split; }

// Workspace bytes of a decode with splits of `split` positions: partial outputs
// [B*H, n_splits, D] fp32 (rounded up to 256 bytes), then their LSEs [B*H, n_splits].
size_t decode_ws_bytes(int B, int H, int cap, int D, int split) {
  const size_t rows = static_cast<size_t>(B) * H;
  const size_t ns = static_cast<size_t>(decode_splits(cap, split));
  const size_t o_bytes = rows * ns * D * sizeof(float);
  return ((o_bytes + 255) & ~static_cast<size_t>(255)) + rows * ns * sizeof(float);
}

// The split size a decode uses: the caller's, or the library's choice.  Measured on B200
// (B16 H32 cap 8192 D128 f16): 128-position splits stream 1.5-2 % faster with one query
// head per kv head; with grouped heads the tensor-core kernel is 2-16 % slower at 128.
int decode_split_for(const flex_decode_params_t* dp, int G) {
  if (dp && dp->split_size != 0) return dp->split_size;
  return G == 1 ? kChunkMin : kChunkMax;
}

constexpr unsigned kStatusSelftestTimeout = 8u;

// One thread waits on a barrier that nothing arrives on, with the bounded wait the
// kernels use; the wait must give up, set the status bit and let the kernel end.
__global__ void selftest_wait_kernel(uint64_t timeout_ns, unsigned* status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  mbar_wait(b, 0, status, kStatusSelftestTimeout, timeout_ns);
}

// Kernel mask kind of a flex_mask_mod_t, or -1.
int mask_kind(int mask_mod_id) {
  switch (mask_mod_id) {
    case FLEX_MASK_NONE: return kMaskNone;
    case FLEX_MASK_CAUSAL:
    case FLEX_MASK_CAUSAL_FAST: return kMaskCausal;
    case FLEX_MASK_SLIDING_WINDOW: return kMaskSliding;
    case FLEX_MASK_KV_LE_Q_PLUS_OFFSET: return kMaskOffset;
    case FLEX_MASK_DOCUMENT: return kMaskDocument;
    case FLEX_MASK_DOCUMENT_CAUSAL: return kMaskDocumentCausal;
  }
  return -1;
}

// The document rules' captured boundaries: present, aligned, of a size that indexes in int64.
flex_status_t check_documents(int mask, const flex_mod_params_t& mp) {
  if (mask != kMaskDocument && mask != kMaskDocumentCausal) return FLEX_OK;
  if (!mp.doc_offsets_q || mp.n_docs < 0 || mp.n_docs > (1 << 24)) return FLEX_ERR_INVALID_ARG;
  if (!aligned4(mp.doc_offsets_q) || (mp.doc_offsets_kv && !aligned4(mp.doc_offsets_kv))) return FLEX_ERR_MISALIGNED;
  return FLEX_OK;
}

MaskArgs mask_args(int mask, const flex_mod_params_t& mp, int Skv) {
  MaskArgs m{Skv, mp.window, mp.offset};
  if (mask == kMaskDocument || mask == kMaskDocumentCausal) {
    m.off_q = mp.doc_offsets_q;
    m.off_kv = mp.doc_offsets_kv ? mp.doc_offsets_kv : mp.doc_offsets_q;
    m.n_docs = mp.n_docs;
  }
  return m;
}

// A block mask's lists: present in pairs, shapes that broadcast over (B, H), 128 x 128
// blocks, key tiles the per-CTA bitmaps can name, 4-byte aligned.
flex_status_t check_block_mask(const flex_block_mask_t& bm, int B, int H, int Sq, int Skv) {
  const bool has_part = bm.kv_num_blocks != nullptr, has_full = bm.full_kv_num_blocks != nullptr;
  if (has_part != (bm.kv_indices != nullptr) || has_full != (bm.full_kv_indices != nullptr))
    return FLEX_ERR_INVALID_ARG;
  if (!has_part && !has_full) return FLEX_ERR_INVALID_ARG;
  if (bm.max_blocks < 1 || (bm.batch != 1 && bm.batch != B) || (bm.heads != 1 && bm.heads != H))
    return FLEX_ERR_INVALID_ARG;
  if (bm.q_block_size != kBM || bm.kv_block_size != kBN) return FLEX_ERR_UNSUPPORTED;
  if ((Skv + kBN - 1) / kBN > kMaxBlockKeyTiles) return FLEX_ERR_UNSUPPORTED;
  const int64_t idx_elems = static_cast<int64_t>(bm.batch) * bm.heads * ((Sq + kBM - 1) / kBM) * bm.max_blocks;
  if (idx_elems > 0x7fffffffLL) return FLEX_ERR_UNSUPPORTED;
  if (!aligned4(bm.kv_num_blocks) || !aligned4(bm.kv_indices) || !aligned4(bm.full_kv_num_blocks) ||
      !aligned4(bm.full_kv_indices))
    return FLEX_ERR_MISALIGNED;
  return FLEX_OK;
}

// Backward workspace: -LSE*log2(e) and -delta per row (rows padded to 128), then, with a
// block mask, the transposed bitmaps (B * Hkv * n_ktiles rows of 2 * tb_words words).
size_t bwd_ws_bytes(int B, int H, int Hkv, int Sq, int Skv, bool blocks) {
  const size_t sq_pad = (static_cast<size_t>(Sq) + kBM - 1) / kBM * kBM;
  size_t bytes = 2 * static_cast<size_t>(B) * H * sq_pad * sizeof(float);
  if (blocks) {
    const size_t nq = (static_cast<size_t>(Sq) + kBM - 1) / kBM, nk = (static_cast<size_t>(Skv) + kBN - 1) / kBN;
    const size_t words = (static_cast<size_t>(H / Hkv) * nq + 31) / 32;
    bytes += static_cast<size_t>(B) * Hkv * nk * 2 * words * sizeof(uint32_t);
  }
  return bytes;
}

// Heads per group of the forward's unit order (unit_coords_of).  Units whose work grows
// with the query position (causal, kv <= q + offset) run heaviest first over groups of
// heads whose K and V (`elem` bytes per element, 32 MiB at most) stay in L2, so that the
// block scheduler's last wave holds the lightest units; other masks run head by head.
// (Measured on B200 against head by head: causal S=2048 +11 %, S=4096 +9 %, S=8192 +7 %,
// GQA D=64 S=4096 +14 %.)
int head_group_for(int mask, int64_t bh, int G, int Skv, int D, int elem) {
  if (mask != kMaskCausal && mask != kMaskOffset) return 1;
  const int64_t kv_head_bytes = static_cast<int64_t>(Skv) * D * elem * 2;
  const int64_t kv_heads = std::max<int64_t>(1, (int64_t{32} << 20) / kv_head_bytes);
  return static_cast<int>(std::min<int64_t>(bh, kv_heads * G));
}

// Shared body of flex_attn_fwd (bm == nullptr) and flex_attn_fwd_block_sparse.
flex_status_t fwd_common(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                         int Sq, int Skv, int D, float scale, int score_mod_id, int mask_mod_id,
                         const flex_mod_params_t* mod_params, const flex_block_mask_t* bm, flex_dtype_t dtype,
                         flex_stream_t stream) {
  if (!q || !k || !v || !o) return FLEX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || H % Hkv != 0) return FLEX_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FLEX_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FLEX_ERR_UNSUPPORTED;
  if (dtype != FLEX_DTYPE_BF16 && dtype != FLEX_DTYPE_F16) return FLEX_ERR_UNSUPPORTED;
  if (score_mod_id != FLEX_SCORE_NONE && score_mod_id != FLEX_SCORE_ALIBI && score_mod_id != FLEX_SCORE_ALIBI_SLOPES)
    return FLEX_ERR_INVALID_ARG;
  const int mask = mask_kind(mask_mod_id);
  if (mask < 0) return FLEX_ERR_INVALID_ARG;
  const flex_mod_params_t zero{};
  const flex_mod_params_t& mp = mod_params ? *mod_params : zero;
  if (mask == kMaskSliding && mp.window < 1) return FLEX_ERR_INVALID_ARG;
  if (score_mod_id == FLEX_SCORE_ALIBI_SLOPES) {
    if (!mp.alibi_slopes) return FLEX_ERR_INVALID_ARG;
    if (!aligned4(mp.alibi_slopes)) return FLEX_ERR_MISALIGNED;
  }
  if (const flex_status_t ds = check_documents(mask, mp); ds != FLEX_OK) return ds;
  // document masks walk per-CTA bitmaps of key tiles, like block masks
  if ((mask == kMaskDocument || mask == kMaskDocumentCausal) && (Skv + kBN - 1) / kBN > kMaxBlockKeyTiles)
    return FLEX_ERR_UNSUPPORTED;
  const bool want_map = (mp.flags & FLEX_FLAG_TILE_MAP) != 0;
  if (want_map && !mp.tile_map_out) return FLEX_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return FLEX_ERR_MISALIGNED;
  if (bm) {
    if (const flex_status_t bs = check_block_mask(*bm, B, H, Sq, Skv); bs != FLEX_OK) return bs;
  }
  const int64_t bh = static_cast<int64_t>(B) * H;
  const int n_qtiles = (Sq + kBM - 1) / kBM;
  const int n_pairs = (n_qtiles + 1) / 2;
  const int64_t n_units = bh * n_pairs;
  if (n_units > 0x7fffffff || static_cast<int64_t>(B) * Hkv > 0x7fffffff) return FLEX_ERR_UNSUPPORTED;

  if (mp.status_out && !aligned4(mp.status_out)) return FLEX_ERR_MISALIGNED;
  unsigned* st = status_for(mp.status_out);
  if (!st) return FLEX_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, dtype, D, Sq, bh) || !make_map(&mk, k, dtype, D, Skv, static_cast<int64_t>(B) * Hkv) ||
      !make_map(&mv, v, dtype, D, Skv, static_cast<int64_t>(B) * Hkv))
    return FLEX_ERR_CUDA;

  FwdParams p{};
  p.o = o;
  p.lse = lse;
  p.tile_map = want_map ? mp.tile_map_out : nullptr;
  p.status = st;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.n_qtiles = n_qtiles;
  p.n_ktiles = (Skv + kBN - 1) / kBN;
  p.n_pairs = n_pairs;
  p.n_units = static_cast<int>(n_units);
  p.bh_total = static_cast<int>(bh);
  p.head_group = bm ? 1 : head_group_for(mask, bh, H / Hkv, Skv, D, 2);
  p.n_full = p.n_items = static_cast<int>(n_units);
  p.n_parts = 1;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Units of uniform work (no mask or a sliding window, no block lists) run in rounds of
  // one CTA per SM: on the persistent kernel when a query tile visits few key tiles (a
  // CTA's fill and drain would otherwise be a large share of its time), else one CTA per
  // unit, which the block scheduler places in waves.  (Measured on B200, 128-row tiles,
  // persistent against per-unit: 3-4 key tiles +15 %, 8 +9 %, 10 +2 %, 16 +4 to +8 %,
  // 32 at D = 64 +7 %, 32 at D = 128 -1 %, 48 and 64 -2 to -5 %, 128 equal.)
  const bool uniform = mask == kMaskNone || mask == kMaskSliding;
  const bool rising = mask == kMaskCausal || mask == kMaskOffset;
  if (!bm && (uniform || rising)) {
    int64_t span = p.n_ktiles;
    if (mask == kMaskSliding)
      span = std::min<int64_t>(span, (static_cast<int64_t>(mp.window) + kBM - 1 + kBN - 1) / kBN + 1);
    const int sms = sm_count();
    if (sms < 1) return FLEX_ERR_CUDA;
    const int64_t grid = n_units < sms ? n_units : sms;
    // Causal-like units run persistent only while every head's K and V fit in L2 at once:
    // then all units form one list, heaviest first, which the kernel's snake order over
    // the CTAs spreads evenly.
    const int64_t kv_bytes = static_cast<int64_t>(B) * Hkv * Skv * D * 2 * 2;
    if (span <= kPersistMaxKeyTiles && (uniform || kv_bytes <= kPersistRisingMaxKvBytes)) {
      p.persist_grid = static_cast<int>(grid);
      if (rising) p.head_group = static_cast<int>(bh);
    }
    if (uniform) {
      // The last round: R = n_units mod grid units would leave grid - R SMs idle.  With
      // R <= grid / 2 their key ranges split into parts (at most 4, at most one per key
      // tile) that fill the round; the last part of each to finish merges them.  (B2 H32
      // S2048: 512 units on 148 SMs take 4 rounds, as long as 592 units did.)  Not with
      // the debug tile map, whose per-tile writes assume whole units.
      const int64_t R = n_units % grid;
      const int64_t parts = R > 0 ? std::min<int64_t>({kMaxParts, grid / R, span}) : 1;
      if (parts >= 2 && !want_map) {
        SplitWorkspace ws{};
        size_t cnt_bytes = 0, ml_bytes = 0;
        if (split_workspace(s, sms, &ws, &cnt_bytes, &ml_bytes)) {
          char* base = static_cast<char*>(ws.base);
          p.part_cnt = reinterpret_cast<unsigned long long*>(base);
          p.part_tag = ws.tag;
          p.part_ml = reinterpret_cast<float2*>(base + cnt_bytes);
          p.part_o = reinterpret_cast<float*>(base + cnt_bytes + ml_bytes);
          p.n_full = static_cast<int>(n_units - R);
          p.n_parts = static_cast<int>(parts);
          p.n_items = static_cast<int>(n_units - R + R * parts);
        }  // else whole units only
      }
    }
  }
  p.scale_log2 = scale * kLog2e;
  p.mask = mask_args(mask, mp, Skv);
  p.slopes = score_mod_id == FLEX_SCORE_ALIBI_SLOPES ? mp.alibi_slopes : nullptr;
  const int score = score_mod_id == FLEX_SCORE_NONE ? kScoreNone : kScoreAlibi;
  const int units = static_cast<int>(n_units);
  if (bm) {
    p.blk_num[0] = bm->kv_num_blocks;
    p.blk_idx[0] = bm->kv_indices;
    p.blk_num[1] = bm->full_kv_num_blocks;
    p.blk_idx[1] = bm->full_kv_indices;
    p.blk_max = bm->max_blocks;
    p.blk_b_stride = bm->batch == 1 ? 0 : bm->heads;
    p.blk_h_stride = bm->heads == 1 ? 0 : 1;
    return D == 128 ? fwd_dispatch<128, true>(dtype, score, mask, mq, mk, mv, p, units, s)
                    : fwd_dispatch<64, true>(dtype, score, mask, mq, mk, mv, p, units, s);
  }
  return D == 128 ? fwd_dispatch<128, false>(dtype, score, mask, mq, mk, mv, p, units, s)
                  : fwd_dispatch<64, false>(dtype, score, mask, mq, mk, mv, p, units, s);
}

}  // namespace
}  // namespace flexattn

using namespace flexattn;

extern "C" {

flex_status_t flex_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                            int Sq, int Skv, int D, float scale, int score_mod_id, int mask_mod_id,
                            const flex_mod_params_t* mod_params, flex_dtype_t dtype, flex_stream_t stream) {
  return fwd_common(q, k, v, o, lse, B, H, Hkv, Sq, Skv, D, scale, score_mod_id, mask_mod_id, mod_params, nullptr,
                    dtype, stream);
}

flex_status_t flex_attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                                         int H, int Hkv, int Sq, int Skv, int D, float scale, int score_mod_id,
                                         int mask_mod_id, const flex_mod_params_t* mod_params,
                                         const flex_block_mask_t* block_mask, flex_dtype_t dtype,
                                         flex_stream_t stream) {
  if (!block_mask) return FLEX_ERR_INVALID_ARG;
  return fwd_common(q, k, v, o, lse, B, H, Hkv, Sq, Skv, D, scale, score_mod_id, mask_mod_id, mod_params,
                    block_mask, dtype, stream);
}

}  // extern "C"

namespace flexattn {
namespace {

// ---------------------------------------------------------------- forward from host buffers

// The built-in alibi slopes of the query heads, computed as the kernels compute them (so a
// chunk that starts at head h0 reads slopes[h0 ..] and gets the same bits).
__global__ void alibi_slope_table_kernel(float* out, int H) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h < H) out[h] = exp2f(-8.0f * static_cast<float>(h + 1) / static_cast<float>(H));
}

// flex_attn_fwd_host splits the work into about kHostChunks chunks and keeps kHostBuffers of
// them on the device: with fewer batches than that, ranges of hc kv heads (and their G
// query heads) of one batch; otherwise runs of bc whole batches (contiguous in every
// tensor, so a run is one forward call over bc batches).
constexpr int kHostChunks = 16;
constexpr int kHostBuffers = 3;

struct HostPlan {
  int per_batch, hc, bc, n, nb;  // chunks per batch, kv heads per chunk, batches per chunk
  size_t q_bytes, kv_bytes, lse_bytes, buf_bytes, slope_off, total;
};

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

HostPlan host_plan(int B, int H, int Hkv, int Sq, int Skv, int D) {
  HostPlan pl{};
  const int G = H / Hkv;
  if (B >= kHostChunks) {  // runs of whole batches
    pl.bc = (B + kHostChunks - 1) / kHostChunks;
    pl.hc = Hkv;
    pl.per_batch = 1;
    pl.n = (B + pl.bc - 1) / pl.bc;
  } else {  // kv-head ranges of one batch
    const int want = std::max(1, std::min(Hkv, (kHostChunks + B - 1) / B));
    pl.bc = 1;
    pl.hc = (Hkv + want - 1) / want;
    pl.per_batch = (Hkv + pl.hc - 1) / pl.hc;
    pl.n = B * pl.per_batch;
  }
  pl.nb = std::min(kHostBuffers, pl.n);
  const size_t heads = static_cast<size_t>(pl.bc) * pl.hc;  // kv heads of one chunk
  pl.q_bytes = align256(heads * G * Sq * D * 2);
  pl.kv_bytes = align256(heads * Skv * D * 2);
  pl.lse_bytes = align256(heads * G * Sq * sizeof(float));
  pl.buf_bytes = 2 * pl.q_bytes + 2 * pl.kv_bytes + pl.lse_bytes;  // Q, K, V, O, LSE
  pl.slope_off = static_cast<size_t>(pl.nb) * pl.buf_bytes;
  pl.total = pl.slope_off + align256(static_cast<size_t>(H) * sizeof(float));
  return pl;
}

// The copy streams and events of the host pipeline, one set per context, created on first
// use and kept for the process's life.  A call holds the set's mutex while it enqueues, so
// every wait on an event is enqueued after that call's record of it.
struct HostPipe {
  unsigned long long ctx;
  cudaStream_t in, out;
  cudaEvent_t start, end, ev_in[kHostBuffers], ev_comp[kHostBuffers], ev_out[kHostBuffers];
  std::mutex mu;
};

HostPipe* host_pipe() {
  static std::vector<HostPipe*> pipes;
  static std::mutex mu;
  unsigned long long id = 0;
  if (!current_context_id(&id)) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  for (HostPipe* hp : pipes)
    if (hp->ctx == id) return hp;
  HostPipe* hp = new HostPipe();
  hp->ctx = id;
  bool ok = cudaStreamCreateWithFlags(&hp->in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&hp->out, cudaStreamNonBlocking) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp->start, cudaEventDisableTiming) == cudaSuccess &&
            cudaEventCreateWithFlags(&hp->end, cudaEventDisableTiming) == cudaSuccess;
  for (int i = 0; ok && i < kHostBuffers; ++i)
    ok = cudaEventCreateWithFlags(&hp->ev_in[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp->ev_comp[i], cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&hp->ev_out[i], cudaEventDisableTiming) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    return nullptr;  // (the partly created set is leaked: this only happens when CUDA fails)
  }
  pipes.push_back(hp);
  return hp;
}

}  // namespace
}  // namespace flexattn

extern "C" {

size_t flex_attn_fwd_host_workspace_size(int B, int H, int Hkv, int Sq, int Skv, int D) {
  if (B < 1 || H < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || H % Hkv != 0 || (D != 64 && D != 128)) return 0;
  return flexattn::host_plan(B, H, Hkv, Sq, Skv, D).total;
}

flex_status_t flex_attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                 int Hkv, int Sq, int Skv, int D, float scale, int score_mod_id, int mask_mod_id,
                                 const flex_mod_params_t* mod_params, flex_dtype_t dtype, void* workspace,
                                 size_t workspace_bytes, flex_stream_t stream) {
  using namespace flexattn;
  if (!q || !k || !v || !o) return FLEX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || H % Hkv != 0) return FLEX_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FLEX_ERR_UNSUPPORTED;
  if (dtype != FLEX_DTYPE_BF16 && dtype != FLEX_DTYPE_F16) return FLEX_ERR_UNSUPPORTED;
  if (score_mod_id != FLEX_SCORE_NONE && score_mod_id != FLEX_SCORE_ALIBI && score_mod_id != FLEX_SCORE_ALIBI_SLOPES)
    return FLEX_ERR_INVALID_ARG;
  const flex_mod_params_t zero{};
  const flex_mod_params_t& mp = mod_params ? *mod_params : zero;
  if (mp.flags & FLEX_FLAG_TILE_MAP) return FLEX_ERR_INVALID_ARG;  // the debug map covers whole calls only
  // the checks each chunk's forward makes again, here before any copy is queued
  if (!(scale > 0.f) || !std::isfinite(scale)) return FLEX_ERR_INVALID_ARG;
  const int mask = mask_kind(mask_mod_id);
  if (mask < 0) return FLEX_ERR_INVALID_ARG;
  if (mask == kMaskSliding && mp.window < 1) return FLEX_ERR_INVALID_ARG;
  if (score_mod_id == FLEX_SCORE_ALIBI_SLOPES) {
    if (!mp.alibi_slopes) return FLEX_ERR_INVALID_ARG;
    if (!aligned4(mp.alibi_slopes)) return FLEX_ERR_MISALIGNED;
  }
  if (const flex_status_t ds = check_documents(mask, mp); ds != FLEX_OK) return ds;
  if ((mask == kMaskDocument || mask == kMaskDocumentCausal) && (Skv + kBN - 1) / kBN > kMaxBlockKeyTiles)
    return FLEX_ERR_UNSUPPORTED;
  if (mp.status_out && !aligned4(mp.status_out)) return FLEX_ERR_MISALIGNED;
  const HostPlan pl = host_plan(B, H, Hkv, Sq, Skv, D);
  if (!workspace || workspace_bytes < pl.total) return FLEX_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FLEX_ERR_MISALIGNED;
  HostPipe* hp = host_pipe();
  if (!hp) return FLEX_ERR_CUDA;
  const int G = H / Hkv;
  const size_t es = 2;  // bytes per element
  char* ws = static_cast<char*>(workspace);
  float* slopes = reinterpret_cast<float*>(ws + pl.slope_off);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(hp->mu);
  flex_status_t rc = FLEX_OK;
  auto cuda_ok = [&rc](cudaError_t e) {
    if (e != cudaSuccess && rc == FLEX_OK) rc = FLEX_ERR_CUDA;
    return e == cudaSuccess;
  };
  // the copy streams start after the work already on the caller's stream
  cuda_ok(cudaEventRecord(hp->start, cs));
  cuda_ok(cudaStreamWaitEvent(hp->in, hp->start, 0));
  cuda_ok(cudaStreamWaitEvent(hp->out, hp->start, 0));
  const float* table = mp.alibi_slopes;
  if (score_mod_id == FLEX_SCORE_ALIBI) {
    alibi_slope_table_kernel<<<(H + 127) / 128, 128, 0, cs>>>(slopes, H);
    cuda_ok(cudaGetLastError());
    table = slopes;
  }
  for (int c = 0; c < pl.n && rc == FLEX_OK; ++c) {
    // batches [b, b + nbat) and, of each, kv heads [hk0, hk0 + nk) (all of them when nbat > 1)
    const int b = (c / pl.per_batch) * pl.bc, nbat = std::min(B, b + pl.bc) - b;
    const int hk0 = (c % pl.per_batch) * pl.hc;
    const int nk = std::min(Hkv, hk0 + pl.hc) - hk0, nh = nk * G, h0 = hk0 * G;
    const int buf = c % pl.nb;
    char* base = ws + static_cast<size_t>(buf) * pl.buf_bytes;
    char* dq = base;
    char* dk = dq + pl.q_bytes;
    char* dv = dk + pl.kv_bytes;
    char* dout = dv + pl.kv_bytes;
    float* dlse = reinterpret_cast<float*>(dout + pl.q_bytes);
    const size_t q_off = (static_cast<size_t>(b) * H + h0) * Sq * D * es,
                 q_len = static_cast<size_t>(nbat) * nh * Sq * D * es;
    const size_t kv_off = (static_cast<size_t>(b) * Hkv + hk0) * Skv * D * es,
                 kv_len = static_cast<size_t>(nbat) * nk * Skv * D * es;
    const size_t l_off = (static_cast<size_t>(b) * H + h0) * Sq,
                 l_len = static_cast<size_t>(nbat) * nh * Sq * sizeof(float);
    // in: this buffer's inputs were read by the forward of chunk c - nb
    if (c >= pl.nb) cuda_ok(cudaStreamWaitEvent(hp->in, hp->ev_comp[buf], 0));
    cuda_ok(cudaMemcpyAsync(dq, static_cast<const char*>(q) + q_off, q_len, cudaMemcpyHostToDevice, hp->in));
    cuda_ok(cudaMemcpyAsync(dk, static_cast<const char*>(k) + kv_off, kv_len, cudaMemcpyHostToDevice, hp->in));
    cuda_ok(cudaMemcpyAsync(dv, static_cast<const char*>(v) + kv_off, kv_len, cudaMemcpyHostToDevice, hp->in));
    cuda_ok(cudaEventRecord(hp->ev_in[buf], hp->in));
    // compute, on the caller's stream: after the inputs, and after chunk c - nb's outputs left
    cuda_ok(cudaStreamWaitEvent(cs, hp->ev_in[buf], 0));
    if (c >= pl.nb) cuda_ok(cudaStreamWaitEvent(cs, hp->ev_out[buf], 0));
    if (rc != FLEX_OK) break;
    flex_mod_params_t cp = mp;
    if (score_mod_id != FLEX_SCORE_NONE) cp.alibi_slopes = table + h0;
    if (cp.doc_offsets_q) cp.doc_offsets_q += static_cast<size_t>(b) * (mp.n_docs + 1);
    if (cp.doc_offsets_kv) cp.doc_offsets_kv += static_cast<size_t>(b) * (mp.n_docs + 1);
    rc = fwd_common(dq, dk, dv, dout, lse ? dlse : nullptr, nbat, nh, nk, Sq, Skv, D, scale,
                    score_mod_id == FLEX_SCORE_NONE ? FLEX_SCORE_NONE : FLEX_SCORE_ALIBI_SLOPES, mask_mod_id, &cp,
                    nullptr, dtype, stream);
    cuda_ok(cudaEventRecord(hp->ev_comp[buf], cs));
    // out: O and LSE of this chunk
    cuda_ok(cudaStreamWaitEvent(hp->out, hp->ev_comp[buf], 0));
    cuda_ok(cudaMemcpyAsync(static_cast<char*>(o) + q_off, dout, q_len, cudaMemcpyDeviceToHost, hp->out));
    if (lse) cuda_ok(cudaMemcpyAsync(lse + l_off, dlse, l_len, cudaMemcpyDeviceToHost, hp->out));
    cuda_ok(cudaEventRecord(hp->ev_out[buf], hp->out));
  }
  // the caller's stream reaches its next work only after every copy (also after an error)
  const bool joined = cudaEventRecord(hp->end, hp->out) == cudaSuccess &&
                      cudaStreamWaitEvent(cs, hp->end, 0) == cudaSuccess &&
                      cudaEventRecord(hp->start, hp->in) == cudaSuccess &&
                      cudaStreamWaitEvent(cs, hp->start, 0) == cudaSuccess;
  if (!joined && rc == FLEX_OK) rc = FLEX_ERR_CUDA;
  return rc;
}

size_t flex_attn_fwd_fp8_workspace_size(int B, int Hkv, int Skv, int D) {
  if (B < 1 || Hkv < 1 || Skv < 1 || (D != 64 && D != 128)) return 0;
  const size_t skv_pad = (static_cast<size_t>(Skv) + 127) / 128 * 128;
  return static_cast<size_t>(B) * Hkv * D * skv_pad;
}

}  // extern "C"

namespace flexattn {
namespace {

// Shared body of flex_attn_fwd_fp8 (bm == nullptr) and flex_attn_fwd_fp8_block_sparse.
flex_status_t fp8_common(const void* q8, const void* k8, const void* v8, void* o, float* lse, int B, int H, int Hkv,
                         int Sq, int Skv, int D, float scale, float descale_q, float descale_k, float descale_v,
                         int score_mod_id, int mask_mod_id, const flex_mod_params_t* mod_params,
                         const flex_block_mask_t* bm, void* workspace, size_t workspace_bytes, flex_stream_t stream) {
  if (!q8 || !k8 || !v8 || !o) return FLEX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || H % Hkv != 0) return FLEX_ERR_INVALID_ARG;
  for (float f : {scale, descale_q, descale_k, descale_v})
    if (!(f > 0.f) || !std::isfinite(f)) return FLEX_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FLEX_ERR_UNSUPPORTED;
  if (score_mod_id != FLEX_SCORE_NONE && score_mod_id != FLEX_SCORE_ALIBI && score_mod_id != FLEX_SCORE_ALIBI_SLOPES)
    return FLEX_ERR_INVALID_ARG;
  const int mask = mask_kind(mask_mod_id);
  if (mask < 0) return FLEX_ERR_INVALID_ARG;
  const flex_mod_params_t zero{};
  const flex_mod_params_t& mp = mod_params ? *mod_params : zero;
  if (mask == kMaskSliding && mp.window < 1) return FLEX_ERR_INVALID_ARG;
  if (score_mod_id == FLEX_SCORE_ALIBI_SLOPES) {
    if (!mp.alibi_slopes) return FLEX_ERR_INVALID_ARG;
    if (!aligned4(mp.alibi_slopes)) return FLEX_ERR_MISALIGNED;
  }
  if (const flex_status_t ds = check_documents(mask, mp); ds != FLEX_OK) return ds;
  if ((mask == kMaskDocument || mask == kMaskDocumentCausal) && (Skv + kBN - 1) / kBN > kMaxBlockKeyTiles)
    return FLEX_ERR_UNSUPPORTED;
  if (bm) {
    if (const flex_status_t bs = check_block_mask(*bm, B, H, Sq, Skv); bs != FLEX_OK) return bs;
  }
  const bool want_map = (mp.flags & FLEX_FLAG_TILE_MAP) != 0;
  if (want_map && !mp.tile_map_out) return FLEX_ERR_INVALID_ARG;
  const size_t need = flex_attn_fwd_fp8_workspace_size(B, Hkv, Skv, D);
  if (!workspace || workspace_bytes < need) return FLEX_ERR_WORKSPACE;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(v8) || !aligned16(o) || !aligned16(workspace) ||
      (lse && !aligned16(lse)))
    return FLEX_ERR_MISALIGNED;
  const int64_t bh = static_cast<int64_t>(B) * H, bhkv = static_cast<int64_t>(B) * Hkv;
  const int n_qtiles = (Sq + kBM - 1) / kBM, n_pairs = (n_qtiles + 1) / 2;
  const int skv_pad = (Skv + 127) / 128 * 128;
  if (bh * n_pairs > 0x7fffffff || bhkv * (skv_pad / 128) > 0x7fffffff) return FLEX_ERR_UNSUPPORTED;
  if (mp.status_out && !aligned4(mp.status_out)) return FLEX_ERR_MISALIGNED;
  unsigned* st = status_for(mp.status_out);
  if (!st) return FLEX_ERR_CUDA;
  Fp8Maps m;
  if (!make_map_u8(&m.q, q8, D, Sq, bh) || !make_map_u8(&m.k, k8, D, Skv, bhkv) ||
      !make_map_u8(&m.vt, workspace, skv_pad, D, bhkv))
    return FLEX_ERR_CUDA;
  Fp8Params p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.tile_map = want_map ? mp.tile_map_out : nullptr;
  p.status = st;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.Skv_pad = skv_pad;
  p.D = D;
  p.n_qtiles = n_qtiles;
  p.n_ktiles = (Skv + kBN - 1) / kBN;
  p.n_pairs = n_pairs;
  p.bh_total = static_cast<int>(bh);
  p.head_group = bm ? 1 : head_group_for(mask, bh, H / Hkv, Skv, D, 1);
  p.scale_log2 = scale * descale_q * descale_k * kLog2e;
  p.descale_v = descale_v;
  p.slopes = score_mod_id == FLEX_SCORE_ALIBI_SLOPES ? mp.alibi_slopes : nullptr;
  p.mask = mask_args(mask, mp, Skv);
  if (bm) {
    p.blocks = VisitLists{{bm->kv_num_blocks, bm->full_kv_num_blocks}, {bm->kv_indices, bm->full_kv_indices},
                          bm->max_blocks, bm->batch == 1 ? 0 : bm->heads, bm->heads == 1 ? 0 : 1};
  }
  const int score = score_mod_id == FLEX_SCORE_NONE ? kScoreNone : kScoreAlibi;
  return fp8_dispatch(score, mask, bm != nullptr, static_cast<const uint8_t*>(v8), static_cast<uint8_t*>(workspace),
                      bhkv, m, p, static_cast<int>(bh * n_pairs), reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace
}  // namespace flexattn

extern "C" {

flex_status_t flex_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, void* o, float* lse, int B, int H,
                                int Hkv, int Sq, int Skv, int D, float scale, float descale_q, float descale_k,
                                float descale_v, int score_mod_id, int mask_mod_id,
                                const flex_mod_params_t* mod_params, void* workspace, size_t workspace_bytes,
                                flex_stream_t stream) {
  return fp8_common(q8, k8, v8, o, lse, B, H, Hkv, Sq, Skv, D, scale, descale_q, descale_k, descale_v, score_mod_id,
                    mask_mod_id, mod_params, nullptr, workspace, workspace_bytes, stream);
}

flex_status_t flex_attn_fwd_fp8_block_sparse(const void* q8, const void* k8, const void* v8, void* o, float* lse,
                                             int B, int H, int Hkv, int Sq, int Skv, int D, float scale,
                                             float descale_q, float descale_k, float descale_v, int score_mod_id,
                                             int mask_mod_id, const flex_mod_params_t* mod_params,
                                             const flex_block_mask_t* block_mask, void* workspace,
                                             size_t workspace_bytes, flex_stream_t stream) {
  if (!block_mask) return FLEX_ERR_INVALID_ARG;
  return fp8_common(q8, k8, v8, o, lse, B, H, Hkv, Sq, Skv, D, scale, descale_q, descale_k, descale_v, score_mod_id,
                    mask_mod_id, mod_params, block_mask, workspace, workspace_bytes, stream);
}

size_t flex_attn_bwd_workspace_size(int B, int H, int Sq) {
  if (B < 1 || H < 1 || Sq < 1) return 0;
  return bwd_ws_bytes(B, H, H, Sq, 1, false);
}

size_t flex_attn_bwd_block_sparse_workspace_size(int B, int H, int Hkv, int Sq, int Skv) {
  if (B < 1 || H < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || H % Hkv != 0) return 0;
  return bwd_ws_bytes(B, H, Hkv, Sq, Skv, true);
}

}  // extern "C"

namespace flexattn {
namespace {

// Shared body of flex_attn_bwd (bm == nullptr) and flex_attn_bwd_block_sparse.
flex_status_t bwd_common(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, int B, int H, int Hkv, int Sq, int Skv,
                         int D, float scale, int score_mod_id, int mask_mod_id, const flex_mod_params_t* mod_params,
                         const flex_block_mask_t* bm, flex_dtype_t dtype, void* workspace, size_t workspace_bytes,
                         flex_stream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FLEX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || Sq < 1 || Skv < 1 || H % Hkv != 0) return FLEX_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FLEX_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FLEX_ERR_UNSUPPORTED;
  if (dtype != FLEX_DTYPE_BF16 && dtype != FLEX_DTYPE_F16) return FLEX_ERR_UNSUPPORTED;
  if (score_mod_id != FLEX_SCORE_NONE && score_mod_id != FLEX_SCORE_ALIBI && score_mod_id != FLEX_SCORE_ALIBI_SLOPES)
    return FLEX_ERR_INVALID_ARG;
  const int mask = mask_kind(mask_mod_id);
  if (mask < 0) return FLEX_ERR_INVALID_ARG;
  const flex_mod_params_t zero{};
  const flex_mod_params_t& mp = mod_params ? *mod_params : zero;
  if (mask == kMaskSliding && mp.window < 1) return FLEX_ERR_INVALID_ARG;
  if (score_mod_id == FLEX_SCORE_ALIBI_SLOPES) {
    if (!mp.alibi_slopes) return FLEX_ERR_INVALID_ARG;
    if (!aligned4(mp.alibi_slopes)) return FLEX_ERR_MISALIGNED;
  }
  if (const flex_status_t ds = check_documents(mask, mp); ds != FLEX_OK) return ds;
  if (bm) {
    if (const flex_status_t bs = check_block_mask(*bm, B, H, Sq, Skv); bs != FLEX_OK) return bs;
  }
  const size_t need = bwd_ws_bytes(B, H, Hkv, Sq, Skv, bm != nullptr);
  if (!workspace || workspace_bytes < need) return FLEX_ERR_WORKSPACE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(workspace) || !aligned4(lse))
    return FLEX_ERR_MISALIGNED;
  const int n_qtiles = (Sq + kBM - 1) / kBM, n_ktiles = (Skv + kBN - 1) / kBN;
  const int64_t bh = static_cast<int64_t>(B) * H, bhkv = static_cast<int64_t>(B) * Hkv;
  if (bh * n_qtiles > 0x7fffffff || bhkv * n_ktiles > 0x7fffffff) return FLEX_ERR_UNSUPPORTED;
  if (mp.status_out && !aligned4(mp.status_out)) return FLEX_ERR_MISALIGNED;
  unsigned* st = status_for(mp.status_out);
  if (!st) return FLEX_ERR_CUDA;
  BwdMaps m;
  if (!make_map(&m.q, q, dtype, D, Sq, bh) || !make_map(&m.o, dout, dtype, D, Sq, bh) ||
      !make_map(&m.k, k, dtype, D, Skv, bhkv) || !make_map(&m.v, v, dtype, D, Skv, bhkv))
    return FLEX_ERR_CUDA;
  BwdParams p{};
  p.o = o;
  p.dout = dout;
  p.lse = lse;
  p.Sq_pad = n_qtiles * kBM;
  p.nlse2 = static_cast<float*>(workspace);
  p.ndelta = p.nlse2 + bh * p.Sq_pad;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.status = st;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.D = D;
  p.n_qtiles = n_qtiles;
  p.n_ktiles = n_ktiles;
  p.q_group = 0;
  p.kv_group = 1;
  if (!bm && (mask == kMaskCausal || mask == kMaskOffset)) {
    // heaviest tiles first over groups of heads whose shared operands stay in L2: the dQ
    // kernel reads K/V of its kv head, the dK/dV kernel Q and dO of the kv head's G heads
    // (measured on B200, causal B2 H32 S8192: see the design notes)
    p.q_group = head_group_for(mask, static_cast<int64_t>(B) * H, H / Hkv, Skv, D, 2);
    const int64_t qdo_bytes = static_cast<int64_t>(H / Hkv) * Sq * D * 2 * 2;
    p.kv_group = static_cast<int>(std::min<int64_t>(static_cast<int64_t>(B) * Hkv,
                                                    std::max<int64_t>(1, (int64_t{32} << 20) / qdo_bytes)));
  }
  p.scale = scale;
  p.scale_log2 = scale * kLog2e;
  p.slopes = score_mod_id == FLEX_SCORE_ALIBI_SLOPES ? mp.alibi_slopes : nullptr;
  p.mask = mask_args(mask, mp, Skv);
  const int score = score_mod_id == FLEX_SCORE_NONE ? kScoreNone : kScoreAlibi;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (bm) {
    p.blk_num[0] = bm->kv_num_blocks;
    p.blk_idx[0] = bm->kv_indices;
    p.blk_num[1] = bm->full_kv_num_blocks;
    p.blk_idx[1] = bm->full_kv_indices;
    p.blk_max = bm->max_blocks;
    p.blk_b_stride = bm->batch == 1 ? 0 : bm->heads;
    p.blk_h_stride = bm->heads == 1 ? 0 : 1;
    p.tbits = reinterpret_cast<uint32_t*>(p.ndelta + bh * p.Sq_pad);
    p.tb_words = (p.G * n_qtiles + 31) / 32;
    return D == 128 ? bwd_dispatch<128, true>(dtype, score, mask, m, p, s)
                    : bwd_dispatch<64, true>(dtype, score, mask, m, p, s);
  }
  return D == 128 ? bwd_dispatch<128, false>(dtype, score, mask, m, p, s)
                  : bwd_dispatch<64, false>(dtype, score, mask, m, p, s);
}

}  // namespace
}  // namespace flexattn

extern "C" {

flex_status_t flex_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                            const void* dout, void* dq, void* dk, void* dv, int B, int H, int Hkv, int Sq, int Skv,
                            int D, float scale, int score_mod_id, int mask_mod_id, const flex_mod_params_t* mod_params,
                            flex_dtype_t dtype, void* workspace, size_t workspace_bytes, flex_stream_t stream) {
  return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, B, H, Hkv, Sq, Skv, D, scale, score_mod_id, mask_mod_id,
                    mod_params, nullptr, dtype, workspace, workspace_bytes, stream);
}

flex_status_t flex_attn_bwd_block_sparse(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                         const void* dout, void* dq, void* dk, void* dv, int B, int H, int Hkv, int Sq,
                                         int Skv, int D, float scale, int score_mod_id, int mask_mod_id,
                                         const flex_mod_params_t* mod_params, const flex_block_mask_t* block_mask,
                                         flex_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                         flex_stream_t stream) {
  if (!block_mask) return FLEX_ERR_INVALID_ARG;
  return bwd_common(q, k, v, o, lse, dout, dq, dk, dv, B, H, Hkv, Sq, Skv, D, scale, score_mod_id, mask_mod_id,
                    mod_params, block_mask, dtype, workspace, workspace_bytes, stream);
}

size_t flex_attn_decode_workspace_size(int B, int H, int Hkv, int cap, int D) {
  if (B < 1 || H < 1 || Hkv < 1 || cap < 1 || D < 1) return 0;
  return decode_ws_bytes(B, H, cap, D, kChunkMin);
}

flex_status_t flex_attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_len,
                               const void* additive_mask, void* o, float* lse, int B, int H, int Hkv, int cap, int D,
                               float scale, flex_dtype_t dtype, void* workspace, size_t workspace_bytes,
                               const flex_decode_params_t* dp, flex_stream_t stream) {
  if (!q || !k_cache || !v_cache || !kv_len || !o) return FLEX_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || Hkv < 1 || cap < 1 || H % Hkv != 0) return FLEX_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FLEX_ERR_INVALID_ARG;
  const int split = decode_split_for(dp, H / Hkv);
  if (split != 128 && split != 256) return FLEX_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FLEX_ERR_UNSUPPORTED;
  if (dtype != FLEX_DTYPE_BF16 && dtype != FLEX_DTYPE_F16) return FLEX_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * Hkv * (H / Hkv) > 65535LL * 8) return FLEX_ERR_UNSUPPORTED;
  const size_t need = decode_ws_bytes(B, H, cap, D, split);
  if (!workspace || workspace_bytes < need) return FLEX_ERR_WORKSPACE;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || !aligned16(workspace) ||
      (lse && !aligned16(lse)) || (additive_mask && !aligned16(additive_mask)) || !aligned16(kv_len))
    return FLEX_ERR_MISALIGNED;
  if (dp && dp->status_out && !aligned4(dp->status_out)) return FLEX_ERR_MISALIGNED;
  unsigned* st = status_for(dp ? dp->status_out : nullptr);
  if (!st) return FLEX_ERR_CUDA;
  DecodeParams p{};
  p.q = q;
  p.k = k_cache;
  p.v = v_cache;
  p.kv_len = kv_len;
  p.mask = additive_mask;
  p.o = o;
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Hkv = Hkv;
  p.G = H / Hkv;
  p.cap = cap;
  p.split = split;
  p.n_splits = decode_splits(cap, split);
  const size_t rows = static_cast<size_t>(B) * H;
  const size_t o_bytes = rows * p.n_splits * D * sizeof(float);
  p.part_o = static_cast<float*>(workspace);
  p.part_lse = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + ((o_bytes + 255) & ~static_cast<size_t>(255)));
  p.status = st;
  p.scale_log2 = scale * kLog2e;
  if (p.G >= 2 && B <= kDtMaxBatch) {
    // grouped heads: the persistent kernel streams the caches in 64-position TMA tiles
    DecodeMaps m;
    if (!make_map(&m.k, k_cache, dtype, D, cap, static_cast<int64_t>(B) * Hkv, kDtKeys) ||
        !make_map(&m.v, v_cache, dtype, D, cap, static_cast<int64_t>(B) * Hkv, kDtKeys))
      return FLEX_ERR_CUDA;
    // the mask tile rides with each K tile through TMA when its rows can be mapped
    m.mask_rows = 0;
    m.m = m.k;
    if (additive_mask != nullptr && cap % 8 == 0) {
      m.mask_rows = p.G < kGqaRows ? p.G : kGqaRows;
      if (!make_map_mask(&m.m, additive_mask, dtype, cap, H, B, m.mask_rows)) return FLEX_ERR_CUDA;
    }
    const int sms = sm_count();
    if (sms < 1) return FLEX_ERR_CUDA;
    const int64_t chunks = static_cast<int64_t>(B) * Hkv * ((p.G + kGqaRows - 1) / kGqaRows) * p.n_splits;
    m.grid = static_cast<int>(chunks < sms ? chunks : sms);
    return decode_dispatch(D, dtype, p, &m, reinterpret_cast<cudaStream_t>(stream));
  }
  const int64_t grid_y = static_cast<int64_t>(B) * Hkv * (p.G >= 2 ? (p.G + kGqaRows - 1) / kGqaRows : 1);
  if (grid_y > 65535) return FLEX_ERR_UNSUPPORTED;
  return decode_dispatch(D, dtype, p, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

flex_status_t flex_attn_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* kv_len, const void* additive_mask, void* o, float* lse,
                                       int B, int H, int Hkv, int cap, int D, float scale, flex_dtype_t dtype,
                                       const flex_decode_params_t* dp, flex_stream_t stream) {
  if (B < 1 || H < 1 || Hkv < 1 || cap < 1 || D < 1) return FLEX_ERR_INVALID_ARG;
  // 256-position splits unless the caller asks otherwise (the smaller workspace)
  flex_decode_params_t use{kChunkMax, nullptr};
  if (dp) {
    use = *dp;
    if (use.split_size == 0) use.split_size = kChunkMax;
  }
  if (use.split_size != 128 && use.split_size != 256) return FLEX_ERR_INVALID_ARG;
  if (decode_ws_bytes(B, H, cap, D, use.split_size) > FLEX_DECODE_STATIC_SCRATCH_BYTES) return FLEX_ERR_WORKSPACE;
  void* scratch = decode_scratch_ptr();
  if (!scratch) return FLEX_ERR_CUDA;
  return flex_attn_decode(q, k_cache, v_cache, kv_len, additive_mask, o, lse, B, H, Hkv, cap, D, scale, dtype,
                          scratch, FLEX_DECODE_STATIC_SCRATCH_BYTES, &use, stream);
}

flex_status_t flex_attn_mask_eval(int mask_mod_id, const flex_mod_params_t* mod_params, int Sq, int Skv,
                                  uint8_t* keep, flex_stream_t stream) {
  if (!keep || Sq < 1 || Skv < 1) return FLEX_ERR_INVALID_ARG;
  const flex_mod_params_t zero{};
  const flex_mod_params_t& mp = mod_params ? *mod_params : zero;
  const int mask = mask_kind(mask_mod_id);
  if (mask < 0) return FLEX_ERR_INVALID_ARG;
  if (const flex_status_t ds = check_documents(mask, mp); ds != FLEX_OK) return ds;
  const MaskArgs m = mask_args(mask, mp, Skv);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t total = static_cast<int64_t>(Sq) * Skv;
  const int grid = static_cast<int>(total / 256 + 1 > 4096 ? 4096 : total / 256 + 1);
  switch (mask_mod_id) {
    case FLEX_MASK_NONE: mask_eval_kernel<kMaskNone><<<grid, 256, 0, s>>>(m, Sq, Skv, keep); break;
    case FLEX_MASK_CAUSAL:
    case FLEX_MASK_CAUSAL_FAST: mask_eval_kernel<kMaskCausal><<<grid, 256, 0, s>>>(m, Sq, Skv, keep); break;
    case FLEX_MASK_SLIDING_WINDOW:
      if (mp.window < 1) return FLEX_ERR_INVALID_ARG;
      mask_eval_kernel<kMaskSliding><<<grid, 256, 0, s>>>(m, Sq, Skv, keep);
      break;
    case FLEX_MASK_KV_LE_Q_PLUS_OFFSET: mask_eval_kernel<kMaskOffset><<<grid, 256, 0, s>>>(m, Sq, Skv, keep); break;
    case FLEX_MASK_DOCUMENT: mask_eval_kernel<kMaskDocument><<<grid, 256, 0, s>>>(m, Sq, Skv, keep); break;
    case FLEX_MASK_DOCUMENT_CAUSAL:
      mask_eval_kernel<kMaskDocumentCausal><<<grid, 256, 0, s>>>(m, Sq, Skv, keep);
      break;
    default: return FLEX_ERR_INVALID_ARG;
  }
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

flex_status_t flex_attn_selftest_wait_timeout(uint32_t timeout_us, flex_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 2000000u) return FLEX_ERR_INVALID_ARG;
  unsigned* st = status_for(nullptr);
  if (!st) return FLEX_ERR_CUDA;
  selftest_wait_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull, st);
  return cudaGetLastError() == cudaSuccess ? FLEX_OK : FLEX_ERR_CUDA;
}

void flex_attn_tile_sizes(int D, int* bm, int* bn) {
  (void)D;
  if (bm) *bm = kBM;
  if (bn) *bn = kBN;
}

flex_status_t flex_attn_device_status(uint32_t* status_out, int reset) {
  if (!status_out) return FLEX_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return FLEX_ERR_CUDA;
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof v) != cudaSuccess) return FLEX_ERR_CUDA;
  *status_out = v;
  if (reset) {
    const unsigned z = 0;
    if (cudaMemcpyToSymbol(g_status, &z, sizeof z) != cudaSuccess) return FLEX_ERR_CUDA;
  }
  return FLEX_OK;
}

const char* flex_status_string(flex_status_t s) {
  switch (s) {
    case FLEX_OK: return "ok";
    case FLEX_ERR_INVALID_ARG: return "invalid argument";
    case FLEX_ERR_UNSUPPORTED: return "unsupported head dim, dtype or size";
    case FLEX_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case FLEX_ERR_WORKSPACE: return "decode workspace missing or too small";
    case FLEX_ERR_CUDA: return "CUDA call failed";
    case FLEX_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

}  // extern "C"
