// Host side of the C ABI declared in include/fp2.h: argument validation, the launch plan,
// workspace sizing, TMA descriptor encoding and kernel launches.  Allocates nothing and
// never synchronises the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>

#include "../../include/fp2.h"
#include "fp2_kernels.h"

namespace {

thread_local std::string g_last_error;

fp2_status fail(fp2_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

fp2_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FP2_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }
// Adaptive splits: at most kMaxPieces pieces per attention launch (the automatic rule typically
// plans 2-3 x SMs), and at most kMaxPieceSplits pieces per row.
constexpr int kMaxPieces = 768;
constexpr int kMaxPieceSplits = 64;
// The automatic mode plans pieces only for launches of fewer row CTAs than 16 waves of a 148-SM
// B200: longer launches balance themselves (rows grow with the query block and run heavy-first),
// and there the plan kernel and the idle piece CTAs would cost a few percent.
constexpr int64_t kAdaptiveRowCtas = 16 * 148;

// f16 operands exist only inside the library (the V side of E4M3 attention); it is no input dtype.
constexpr fp2_dtype kOperandF16 = static_cast<fp2_dtype>(100);

int elt_bytes(fp2_dtype t) { return t == FP2_F32 ? 4 : ((t == FP2_BF16 || t == kOperandF16) ? 2 : 1); }

// Testing hooks set through fp2_debug_set (process-wide; read when attention launches).
std::atomic<int64_t> g_wait_limit_ns{0};     // 0: the default limit of 1 s
std::atomic<int64_t> g_withhold_k_tile{-1};  // -1: every load is issued
std::atomic<int64_t> g_miscount_load{-1};    // -1: every load is counted once (checked builds)

// Everything derived from (problem, params) on the host.
struct Ctx {
  Fp2Plan plan;
  int elt = 0, G = 0, W = 0;
  int64_t T = 0, Tk = 0, total_blocks = 0, total_k_blocks = 0, rows = 0, cap = 0;
  float scale = 0.f;
  fp2_workspace ws{};
  size_t off_bitmask = 0, off_counts = 0;  // inside scratch
  int NT = 1, parts = 1, splits = 1;        // attention launch shape
  size_t off_opart = 0, off_lsepart = 0;    // KV-split partials inside scratch (splits > 1)
  // Adaptive splits (splits == 1): up to `pieces` pieces of long rows, planned on the device.
  int pieces = 0, piece_tiles = 0;          // piece capacity; forced piece size (0 = automatic)
  size_t off_item0 = 0, off_items = 0, off_nitems = 0, off_pcnt = 0, off_oslot = 0, off_lslot = 0;
  // fp2_prefill carve-outs (offsets after scratch_bytes)
  size_t off_qbar = 0, off_kbar = 0, off_vbar = 0, off_kbm = 0, off_vbm = 0, off_v16 = 0, off_rowptr = 0,
         off_colidx = 0;
};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fp2_status validate(const fp2_problem* p, const fp2_sparse_params* s, Ctx& c) {
  if (p == nullptr || s == nullptr) return fail(FP2_ERR_INVALID_ARG, "problem and params must not be NULL");
  if (p->num_seqs < 1 || p->num_seqs > FP2_MAX_SEQS)
    return fail(FP2_ERR_UNSUPPORTED, "num_seqs must be in [1, FP2_MAX_SEQS]");
  if (p->cu_seqlens_q_host == nullptr) return fail(FP2_ERR_INVALID_ARG, "cu_seqlens_q_host is NULL");
  if (p->dtype != FP2_F32 && p->dtype != FP2_BF16 && p->dtype != FP2_E4M3)
    return fail(FP2_ERR_INVALID_ARG, "unknown dtype");
  if (p->num_q_heads <= 0 || p->num_kv_heads <= 0 || p->num_q_heads % p->num_kv_heads != 0)
    return fail(FP2_ERR_INVALID_ARG, "num_q_heads must be a positive multiple of num_kv_heads");
  c.G = p->num_q_heads / p->num_kv_heads;
  if (c.G > 32) return fail(FP2_ERR_UNSUPPORTED, "GQA group size above 32");
  if (p->head_dim != 64 && p->head_dim != 128) return fail(FP2_ERR_UNSUPPORTED, "head_dim must be 64 or 128");
  if (p->dtype == FP2_F32 && p->head_dim != 64) return fail(FP2_ERR_UNSUPPORTED, "F32 inputs need head_dim 64");
  if (p->dtype == FP2_E4M3 && p->head_dim != 128) return fail(FP2_ERR_UNSUPPORTED, "E4M3 inputs need head_dim 128");
  if (s->block_size != 64 && s->block_size != 128) return fail(FP2_ERR_UNSUPPORTED, "block_size must be 64 or 128");
  if (!(s->alpha >= 0.f && s->alpha <= 1.f)) return fail(FP2_ERR_INVALID_ARG, "alpha must be in [0, 1]");
  if (s->sink_blocks < 0 || s->window_blocks < 0 || s->last_n_blocks < 0 || s->min_sparse_len < 0)
    return fail(FP2_ERR_INVALID_ARG, "sink/window/last_n/min_sparse_len must be >= 0");
  if (s->kv_splits < -FP2_MAX_BLOCKS || s->kv_splits > 64)
    return fail(FP2_ERR_INVALID_ARG, "kv_splits must be in [-FP2_MAX_BLOCKS, 64]");
  if (!(p->softmax_scale >= 0.f) || !std::isfinite(p->softmax_scale))
    return fail(FP2_ERR_INVALID_ARG, "softmax_scale must be finite and >= 0");
  for (float d : {p->q_descale, p->k_descale, p->v_descale})
    if (!(d > 0.f) || !std::isfinite(d)) return fail(FP2_ERR_INVALID_ARG, "descale factors must be finite and > 0");
  c.elt = elt_bytes(p->dtype);
  const int B = s->block_size, D = p->head_dim, Hq = p->num_q_heads, Hkv = p->num_kv_heads;

  const int32_t* cq = p->cu_seqlens_q_host;
  const int32_t* ck = p->cu_seqlens_k_host ? p->cu_seqlens_k_host : cq;
  if (cq[0] != 0 || ck[0] != 0) return fail(FP2_ERR_INVALID_ARG, "cu_seqlens must start at 0");
  Fp2Plan& P = c.plan;
  std::memset(&P, 0, sizeof(P));
  P.num_seqs = p->num_seqs;
  int64_t T = 0, Tk = 0, blocks = 0, kblocks = 0, cap = 0;
  int max_nblk = 0, max_k_nblk = 0;
  for (int r = 0; r < p->num_seqs; ++r) {
    const int64_t Lq = static_cast<int64_t>(cq[r + 1]) - cq[r];
    const int64_t Lk = static_cast<int64_t>(ck[r + 1]) - ck[r];
    if (Lq < 0 || Lk < 0) return fail(FP2_ERR_INVALID_ARG, "cu_seqlens must be non-decreasing");
    if (Lk < Lq) return fail(FP2_ERR_INVALID_ARG, "kv_len must be >= q_len for every sequence");
    if ((Lk - Lq) % B != 0)
      return fail(FP2_ERR_UNSUPPORTED, "a query chunk must start on a block boundary (kv_len - q_len % B != 0)");
    const int64_t N = (Lq + B - 1) / B;
    const int64_t pre = (Lk - Lq) / B;
    const int64_t Nk = pre + N;
    if (Nk > FP2_MAX_BLOCKS) return fail(FP2_ERR_UNSUPPORTED, "a sequence has more than FP2_MAX_BLOCKS key blocks");
    P.tok_off[r] = cq[r];
    P.len[r] = static_cast<int32_t>(Lq);
    P.blk_off[r] = static_cast<int32_t>(blocks);
    P.nblk[r] = static_cast<int32_t>(N);
    P.k_tok_off[r] = ck[r];
    P.k_blk_off[r] = static_cast<int32_t>(kblocks);
    P.pre_blk[r] = static_cast<int32_t>(pre);
    T += Lq;
    Tk += Lk;
    blocks += N;
    kblocks += Nk;
    cap += static_cast<int64_t>(Hkv) * (N * pre + N * (N + 1) / 2);  // sum_i (pre + i + 1)
    max_nblk = std::max<int>(max_nblk, static_cast<int>(N));
    max_k_nblk = std::max<int>(max_k_nblk, static_cast<int>(Nk));
  }
  if (T != cq[p->num_seqs] || Tk != ck[p->num_seqs]) return fail(FP2_ERR_INVALID_ARG, "cu_seqlens inconsistent");
  if (Tk >= (int64_t(1) << 31) || cap >= (int64_t(1) << 31) || kblocks * Hkv >= (int64_t(1) << 31))
    return fail(FP2_ERR_UNSUPPORTED, "problem too large for 32-bit token / index offsets");
  P.total_tokens = static_cast<int32_t>(T);
  P.total_blocks = static_cast<int32_t>(blocks);
  P.total_k_tokens = static_cast<int32_t>(Tk);
  P.total_k_blocks = static_cast<int32_t>(kblocks);
  P.max_nblk = max_nblk;
  P.max_k_nblk = max_k_nblk;
  for (int r = 0; r < p->num_seqs; ++r) P.sorted[r] = static_cast<int16_t>(r);
  std::stable_sort(P.sorted, P.sorted + p->num_seqs, [&](int16_t x, int16_t y) { return P.nblk[x] > P.nblk[y]; });
  // Heavy-first work lists: per sorted position k, the items (per unit of width) of the sequences
  // before it, for tiles of one query block and of the discovery tile.
  P.disc_tile = std::max(1, 128 / c.G);
  for (int t = 0; t < 2; ++t) {
    const int tile = t == 0 ? 1 : P.disc_tile;
    int32_t* lb = t == 0 ? P.lvl_base1 : P.lvl_base_t;
    int64_t base = 0;
    for (int k = 0; k < p->num_seqs; ++k) {
      lb[k] = static_cast<int32_t>(base);
      const int64_t hi = (P.nblk[P.sorted[k]] + tile - 1) / tile;
      const int64_t lo = k + 1 < p->num_seqs ? (P.nblk[P.sorted[k + 1]] + tile - 1) / tile : 0;
      base += (hi - lo) * (k + 1);
    }
    lb[p->num_seqs] = static_cast<int32_t>(base);
  }
  c.T = T;
  c.Tk = Tk;
  c.total_blocks = blocks;
  c.total_k_blocks = kblocks;
  c.rows = blocks * Hkv;
  c.cap = cap;
  c.W = std::max(1, (max_k_nblk + 31) / 32);
  c.scale = p->softmax_scale > 0.f ? p->softmax_scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));

  // Tensors (only checked when there is data to read).
  if (T > 0) {
    if (p->q == nullptr || p->k == nullptr || p->v == nullptr) return fail(FP2_ERR_INVALID_ARG, "q/k/v must not be NULL");
    if (!aligned16(p->q) || !aligned16(p->k) || !aligned16(p->v))
      return fail(FP2_ERR_INVALID_ARG, "q/k/v must be 16-byte aligned");
    if (p->q_stride_tok < static_cast<int64_t>(Hq) * D || p->kv_stride_tok < static_cast<int64_t>(Hkv) * D)
      return fail(FP2_ERR_INVALID_ARG, "token strides must be >= heads * head_dim");
    if ((p->q_stride_tok * c.elt) % 16 != 0 || (p->kv_stride_tok * c.elt) % 16 != 0)
      return fail(FP2_ERR_INVALID_ARG, "token strides must be multiples of 16 bytes");
    if (p->page_table != nullptr) {
      const int ps = p->page_size;
      if (ps < 16 || (ps & (ps - 1)) != 0) return fail(FP2_ERR_UNSUPPORTED, "page_size must be a power of two >= 16");
      if (p->num_pages <= 0 || static_cast<int64_t>(p->num_pages) * ps >= (int64_t(1) << 31))
        return fail(FP2_ERR_INVALID_ARG, "num_pages out of range");
      for (int r = 0; r < p->num_seqs; ++r)
        if ((P.pre_blk[r] * B + P.len[r] + ps - 1) / ps > p->max_pages_per_seq)
          return fail(FP2_ERR_INVALID_ARG, "max_pages_per_seq too small for a sequence");
    }
  }

  fp2_workspace& w = c.ws;
  w.total_tokens = T;
  w.total_kv_tokens = Tk;
  w.total_q_blocks = blocks;
  w.total_kv_blocks = kblocks;
  w.index_rows = c.rows;
  w.col_capacity = cap;
  w.qbar_bytes = static_cast<size_t>(blocks) * Hq * D * 4;
  w.kbar_bytes = static_cast<size_t>(kblocks) * Hkv * D * 4;
  w.vbar_bytes = w.kbar_bytes;
  w.kbar_mma_bytes = static_cast<size_t>(kblocks) * Hkv * D * c.elt;
  // The V-side operands of the PV product are f16 for E4M3 inputs (pooled vbar and the V copy).
  const bool e4 = p->dtype == FP2_E4M3;
  w.vbar_mma_bytes = static_cast<size_t>(kblocks) * Hkv * D * (e4 ? 2 : c.elt);
  w.v16_bytes = e4 ? static_cast<size_t>(Tk) * Hkv * D * 2 : 0;
  w.row_ptr_bytes = static_cast<size_t>(c.rows + 1) * 4;
  w.col_idx_bytes = static_cast<size_t>(std::max<int64_t>(cap, 1)) * 4;
  // Attention launch shape: M tiles of 128 packed rows, two per CTA when the group fills them.
  const int mtiles = (c.G * B + 127) / 128;
  c.NT = mtiles >= 2 ? 2 : 1;
  c.parts = (mtiles + c.NT - 1) / c.NT;
  const int64_t row_ctas = c.rows * c.parts;
  if (s->kv_splits > 0)
    c.splits = s->kv_splits;
  else if (s->kv_splits < 0)
    c.splits = 1;
  else
    c.splits = row_ctas >= 296 ? 1 : static_cast<int>(std::min<int64_t>(8, (296 + std::max<int64_t>(row_ctas, 1) - 1) /
                                                                                   std::max<int64_t>(row_ctas, 1)));
  // Rows whose key-tile count is far above the launch's share per SM are cut into pieces planned
  // on the device (kv_splits < 0: pieces of at most -kv_splits tiles; 0 with many rows: automatic).
  if (c.splits == 1 && (s->kv_splits < 0 || (s->kv_splits == 0 && row_ctas < kAdaptiveRowCtas))) {
    c.piece_tiles = s->kv_splits < 0 ? -s->kv_splits : 0;
    c.pieces = static_cast<int>(std::min<int64_t>(kMaxPieces, row_ctas * kMaxPieceSplits));
  }
  c.off_bitmask = FP2_SCRATCH_STATUS_BYTES;
  c.off_counts = c.off_bitmask + align_up(static_cast<size_t>(c.rows) * c.W * 4);
  w.scratch_bytes = c.off_counts + align_up(static_cast<size_t>(c.rows) * 4);
  w.discover_scratch_bytes = w.scratch_bytes;
  if (c.splits > 1) {
    c.off_opart = w.scratch_bytes;
    c.off_lsepart = c.off_opart + align_up(static_cast<size_t>(c.splits) * T * Hq * D * 4);
    w.scratch_bytes = c.off_lsepart + align_up(static_cast<size_t>(c.splits) * Hq * T * 4);
  }
  if (c.pieces > 0) {
    const size_t prow = static_cast<size_t>(c.NT) * 128;  // packed rows of one piece
    c.off_item0 = w.scratch_bytes;
    c.off_items = c.off_item0 + align_up(static_cast<size_t>(c.rows) * 4);
    c.off_nitems = c.off_items + align_up(static_cast<size_t>(c.pieces) * 8);
    c.off_pcnt = c.off_nitems + align_up(4);
    c.off_oslot = c.off_pcnt + align_up(static_cast<size_t>(c.pieces) * 2 * 4);
    c.off_lslot = c.off_oslot + align_up(static_cast<size_t>(c.pieces) * prow * D * 4);
    w.scratch_bytes = c.off_lslot + align_up(static_cast<size_t>(c.pieces) * prow * 4);
  }
  size_t o = w.scratch_bytes;
  c.off_qbar = o;   o += align_up(w.qbar_bytes);
  c.off_kbar = o;   o += align_up(w.kbar_bytes);
  c.off_vbar = o;   o += align_up(w.vbar_bytes);
  c.off_kbm = o;    o += align_up(w.kbar_mma_bytes);
  c.off_vbm = o;    o += align_up(w.vbar_mma_bytes);
  c.off_v16 = o;    o += align_up(w.v16_bytes);
  c.off_rowptr = o; o += align_up(w.row_ptr_bytes);
  c.off_colidx = o; o += align_up(w.col_idx_bytes);
  w.prefill_scratch_bytes = o;
  return FP2_OK;
}

// ---------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D map over a token-major tensor: dims {d, heads, rows}, box {128B/elt, 1, box_rows}, 128B swizzle.
// mn_major_32b: the tile feeds the MMA as an MN-major 32-bit operand (f32 V), which needs the
// 32-byte-chunk flavour of the 128-byte swizzle.
fp2_status encode_3d(CUtensorMap* m, fp2_dtype dt, const void* base, int D, int heads, int64_t rows,
                     int64_t row_stride_elems, int box_rows, bool mn_major_32b = false) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return fail(FP2_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const int elt = elt_bytes(dt);
  const CUtensorMapDataType t = dt == FP2_F32       ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                : dt == FP2_BF16    ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                : dt == kOperandF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(std::max<int64_t>(rows, 1))};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * elt, static_cast<cuuint64_t>(row_stride_elems) * elt};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elt), 1u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(m, t, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        mn_major_32b ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FP2_ERR_CUDA, "cuTensorMapEncodeTiled failed with CUresult " + std::to_string(r));
  return FP2_OK;
}

uint32_t* status_ptr(void* scratch) { return static_cast<uint32_t*>(scratch); }

fp2_status check_scratch(const void* scratch, size_t have, size_t need) {
  if (scratch == nullptr) return fail(FP2_ERR_INVALID_ARG, "scratch is NULL");
  if ((reinterpret_cast<uintptr_t>(scratch) & (kAlign - 1)) != 0)
    return fail(FP2_ERR_INVALID_ARG, "scratch must be 256-byte aligned");
  if (have < need)
    return fail(FP2_ERR_WORKSPACE_TOO_SMALL,
                "scratch_bytes " + std::to_string(have) + " < required " + std::to_string(need));
  return FP2_OK;
}

// need_q: qbar is read or written; need_v16: the E4M3 f16 copy of V is read or written.
fp2_status check_pooled(const fp2_pooled* pl, bool need_q, bool need_v16) {
  if (pl == nullptr) return fail(FP2_ERR_INVALID_ARG, "pooled is NULL");
  if ((need_q && pl->qbar == nullptr) || pl->kbar == nullptr || pl->vbar == nullptr || pl->kbar_mma == nullptr ||
      pl->vbar_mma == nullptr)
    return fail(FP2_ERR_INVALID_ARG, "pooled buffers must not be NULL");
  if (need_v16 && pl->v16 == nullptr) return fail(FP2_ERR_INVALID_ARG, "pooled->v16 must not be NULL for E4M3 inputs");
  const void* bufs[6] = {pl->qbar, pl->kbar, pl->vbar, pl->kbar_mma, pl->vbar_mma, need_v16 ? pl->v16 : nullptr};
  for (const void* q : bufs)
    if (q != nullptr && !aligned16(q)) return fail(FP2_ERR_INVALID_ARG, "pooled buffers must be 16-byte aligned");
  return FP2_OK;
}

fp2_status check_index(const fp2_index* ix, const Ctx& c) {
  if (ix == nullptr || ix->row_ptr == nullptr || ix->col_idx == nullptr)
    return fail(FP2_ERR_INVALID_ARG, "index buffers must not be NULL");
  if (ix->col_capacity < 0) return fail(FP2_ERR_INVALID_ARG, "col_capacity must be >= 0");
  (void)c;
  return FP2_OK;
}

fp2_status run_pool(const fp2_problem* p, const fp2_sparse_params* s, const Ctx& c, const fp2_pooled* pl,
                    void* scratch, cudaStream_t st) {
  fp2::PoolArgs a{};
  a.q = p->q;
  a.k = p->k;
  a.v = p->v;
  a.q_stride = p->q_stride_tok;
  a.kv_stride = p->kv_stride_tok;
  a.page_table = p->page_table;
  a.page_size = p->page_size;
  a.max_pages = p->max_pages_per_seq;
  a.num_pages = p->num_pages;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.D = p->head_dim;
  a.B = s->block_size;
  a.q_descale = p->q_descale;
  a.k_descale = p->k_descale;
  a.v_descale = p->v_descale;
  a.qbar = pl->qbar;
  a.kbar = pl->kbar;
  a.vbar = pl->vbar;
  a.kbar_mma = pl->kbar_mma;
  a.vbar_mma = pl->vbar_mma;
  a.v16 = p->dtype == FP2_E4M3 ? pl->v16 : nullptr;
  a.kv_prefix_pooled = p->kv_prefix_pooled ? 1 : 0;
  a.status = status_ptr(scratch);
  const cudaError_t e = fp2::launch_pool(p->dtype, a, c.plan, st);
  return e == cudaSuccess ? FP2_OK : cuda_fail(e, "pool kernel launch");
}

fp2_status run_discover(const fp2_problem* p, const fp2_sparse_params* s, const Ctx& c, const fp2_pooled* pl,
                        const fp2_index* ix, void* scratch, cudaStream_t st) {
  fp2::DiscArgs a{};
  a.qbar = pl->qbar;
  a.kbar = pl->kbar;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = c.G;
  a.D = p->head_dim;
  a.scale = c.scale;
  a.dense_all = s->alpha <= 0.f ? 1 : 0;
  a.ln_alpha = s->alpha > 0.f ? static_cast<float>(std::log(static_cast<double>(s->alpha))) : 0.f;
  a.sink = s->sink_blocks;
  a.window = s->window_blocks;
  a.last_n = s->last_n_blocks;
  a.min_sparse_len = s->min_sparse_len;
  // One CTA computes the 128 score rows (query block, head) of TI = 128 / G query blocks.
  const int TI = c.plan.disc_tile;
  a.TI = TI;
  a.W = c.W;
  a.bitmask = reinterpret_cast<uint32_t*>(static_cast<char*>(scratch) + c.off_bitmask);
  a.counts = reinterpret_cast<int32_t*>(static_cast<char*>(scratch) + c.off_counts);
  a.status = status_ptr(scratch);
  int64_t items = 0;
  for (int r = 0; r < c.plan.num_seqs; ++r) items += static_cast<int64_t>((c.plan.nblk[r] + TI - 1) / TI) * a.Hkv;
  if (items == 0) return FP2_OK;
  const cudaError_t e = fp2::launch_discover(a, c.plan, items, c.rows, ix->row_ptr, ix->col_idx, ix->col_capacity, st);
  return e == cudaSuccess ? FP2_OK : cuda_fail(e, "discover kernels launch");
}

fp2_status run_attend(const fp2_problem* p, const fp2_sparse_params* s, const Ctx& c, const fp2_pooled* pl,
                      const fp2_index* ix, void* out, float* lse, void* scratch, cudaStream_t st) {
  const int B = s->block_size, D = p->head_dim;
  if (fp2::attention_smem_bytes(p->dtype, D, B) == 0)
    return fail(FP2_ERR_UNSUPPORTED, "no attention kernel for this (dtype, head_dim, block_size)");
  fp2::AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  fp2_status st2;
  const bool paged = p->page_table != nullptr;
  if ((st2 = encode_3d(&a.tm_q, p->dtype, p->q, D, p->num_q_heads, c.T, p->q_stride_tok, B)) != FP2_OK) return st2;
  const int64_t kv_rows = paged ? static_cast<int64_t>(p->num_pages) * p->page_size : c.Tk;
  const int kv_box = paged ? std::min(B, p->page_size) : B;
  if ((st2 = encode_3d(&a.tm_k, p->dtype, p->k, D, p->num_kv_heads, kv_rows, p->kv_stride_tok, kv_box)) != FP2_OK)
    return st2;
  const bool v32 = p->dtype == FP2_F32;
  const bool e4 = p->dtype == FP2_E4M3;
  // E4M3: the PV operand is the f16 copy of V written by fp2_pool (contiguous rows in key-token
  // order even for a paged cache) and the f16 pooled vbar.
  a.v_contig = e4 ? 1 : 0;
  if (e4) {
    if ((st2 = encode_3d(&a.tm_v, kOperandF16, pl->v16, D, p->num_kv_heads, c.Tk,
                         static_cast<int64_t>(p->num_kv_heads) * D, B)) != FP2_OK)
      return st2;
  } else if ((st2 = encode_3d(&a.tm_v, p->dtype, p->v, D, p->num_kv_heads, kv_rows, p->kv_stride_tok, kv_box, v32)) !=
             FP2_OK) {
    return st2;
  }
  const int64_t hd = static_cast<int64_t>(p->num_kv_heads) * D;
  if ((st2 = encode_3d(&a.tm_kb, p->dtype, pl->kbar_mma, D, p->num_kv_heads, c.total_k_blocks, hd, B)) != FP2_OK)
    return st2;
  if ((st2 = encode_3d(&a.tm_vb, e4 ? kOperandF16 : p->dtype, pl->vbar_mma, D, p->num_kv_heads, c.total_k_blocks, hd,
                       B, v32)) != FP2_OK)
    return st2;
  // Output tiles of full blocks go out through TMA stores (16-byte aligned output, no KV split);
  // everything else through per-thread stores.
  if (c.splits == 1 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
    const fp2_dtype odt = p->dtype == FP2_F32 ? FP2_F32 : FP2_BF16;
    a.o_tma = encode_3d(&a.tm_o, odt, out, D, p->num_q_heads, c.T, static_cast<int64_t>(p->num_q_heads) * D, B) ==
                      FP2_OK
                  ? 1
                  : 0;
  }
  a.row_ptr = ix->row_ptr;
  a.col_idx = ix->col_idx;
  a.page_table = p->page_table;
  a.page_size = p->page_size;
  a.max_pages = p->max_pages_per_seq;
  a.num_pages = p->num_pages;
  a.out = out;
  a.lse = lse;
  a.Hq = p->num_q_heads;
  a.Hkv = p->num_kv_heads;
  a.G = c.G;
  a.NT = c.NT;
  a.parts = c.parts;
  a.splits = c.splits;
  a.o_part = c.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(scratch) + c.off_opart) : nullptr;
  a.lse_part = c.splits > 1 ? reinterpret_cast<float*>(static_cast<char*>(scratch) + c.off_lsepart) : nullptr;
  char* sc = static_cast<char*>(scratch);
  a.adapt = c.pieces;
  a.row_item0 = c.pieces ? reinterpret_cast<int32_t*>(sc + c.off_item0) : nullptr;
  a.items = c.pieces ? reinterpret_cast<int2*>(sc + c.off_items) : nullptr;
  a.n_items = c.pieces ? reinterpret_cast<int32_t*>(sc + c.off_nitems) : nullptr;
  a.piece_cnt = c.pieces ? reinterpret_cast<int32_t*>(sc + c.off_pcnt) : nullptr;
  a.o_slot = c.pieces ? reinterpret_cast<float*>(sc + c.off_oslot) : nullptr;
  a.lse_slot = c.pieces ? reinterpret_cast<float*>(sc + c.off_lslot) : nullptr;
  a.sm_scale_log2 = static_cast<float>(static_cast<double>(c.scale) * 1.4426950408889634 *
                                       static_cast<double>(p->q_descale) * static_cast<double>(p->k_descale));
  a.v_descale = p->v_descale;
  a.log2_blk = static_cast<float>(std::log2(static_cast<double>(B)));
  a.mean_correction = s->mean_correction ? 1 : 0;
  a.total_tokens = static_cast<int>(c.T);
  a.status = status_ptr(scratch);
  const int64_t lim = g_wait_limit_ns.load();
  a.wait_limit_ns = lim > 0 ? static_cast<uint64_t>(lim) : 1000000000ull;
  a.withhold_k_tile = static_cast<int>(g_withhold_k_tile.load());
  a.miscount_load = static_cast<int>(g_miscount_load.load());
  {
    int dev = 0, nsm = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    a.num_sms = nsm;
  }
  const int64_t row_items = c.total_blocks * p->num_kv_heads * a.parts * a.splits;
  if (row_items == 0) return FP2_OK;
  cudaError_t e;
  if (c.pieces > 0) {
    e = fp2::launch_split_plan(a, c.plan, c.rows, B, c.piece_tiles, st);
    if (e != cudaSuccess) return cuda_fail(e, "split plan kernel launch");
  }
  e = fp2::launch_attention(p->dtype, D, B, a, c.plan, row_items + a.adapt, st);
  if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
  if (c.splits > 1) {
    e = fp2::launch_combine(p->dtype, D, a.o_part, a.lse_part, c.splits, static_cast<int>(c.T), p->num_q_heads, out,
                            lse, st);
    if (e != cudaSuccess) return cuda_fail(e, "split combine kernel launch");
  }
  return FP2_OK;
}

fp2_status clear_status(void* scratch, cudaStream_t st) {
  const cudaError_t e = cudaMemsetAsync(scratch, 0, FP2_SCRATCH_STATUS_BYTES, st);
  return e == cudaSuccess ? FP2_OK : cuda_fail(e, "status reset");
}

}  // namespace

namespace fp2 {

cudaError_t ensure_dynamic_smem(const void* kernel, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, int> granted;  // (kernel, device) -> bytes
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  int& have = granted[{kernel, dev}];
  if (have >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) have = bytes;
  return e;
}

}  // namespace fp2

// Used by fp2_noalloc.cu only: discovery into a caller-supplied scratch region of a fixed capacity,
// optionally copying the device status word to status_dev afterwards.
namespace fp2_internal {

fp2_status set_error(fp2_status s, const char* msg) { return fail(s, msg); }

fp2_status discover_fixed_scratch(const fp2_problem* problem, const fp2_sparse_params* params,
                                  const fp2_pooled* pooled, const fp2_index* index, void* scratch,
                                  size_t capacity, uint32_t* status_dev, cudaStream_t st) {
  Ctx c;
  fp2_status s;
  if ((s = validate(problem, params, c)) != FP2_OK) return s;
  if (c.ws.discover_scratch_bytes > capacity)
    return fail(FP2_ERR_UNSUPPORTED, "problem needs " + std::to_string(c.ws.discover_scratch_bytes) +
                                         " bytes of discovery scratch; the static buffer holds " +
                                         std::to_string(capacity));
  if ((s = check_pooled(pooled, true, false)) != FP2_OK) return s;
  if ((s = check_index(index, c)) != FP2_OK) return s;
  if ((s = clear_status(scratch, st)) != FP2_OK) return s;
  if (c.T > 0 && (s = run_discover(problem, params, c, pooled, index, scratch, st)) != FP2_OK) return s;
  if (status_dev != nullptr) {
    const cudaError_t e = cudaMemcpyAsync(status_dev, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "status copy");
  }
  return FP2_OK;
}

}  // namespace fp2_internal

extern "C" {

fp2_status fp2_workspace_query(const fp2_problem* problem, const fp2_sparse_params* params, fp2_workspace* out) {
  if (out == nullptr) return fail(FP2_ERR_INVALID_ARG, "out is NULL");
  Ctx c;
  const fp2_status s = validate(problem, params, c);
  if (s != FP2_OK) return s;
  *out = c.ws;
  g_last_error.clear();
  return FP2_OK;
}

fp2_status fp2_workspace_size(const fp2_problem* problem, const fp2_sparse_params* params, size_t* pooled_bytes,
                              size_t* index_bytes, size_t* scratch_bytes) {
  Ctx c;
  const fp2_status s = validate(problem, params, c);
  if (s != FP2_OK) return s;
  const fp2_workspace& w = c.ws;
  if (pooled_bytes != nullptr)
    *pooled_bytes = align_up(w.qbar_bytes) + align_up(w.kbar_bytes) + align_up(w.vbar_bytes) +
                    align_up(w.kbar_mma_bytes) + align_up(w.vbar_mma_bytes) + align_up(w.v16_bytes);
  if (index_bytes != nullptr) *index_bytes = align_up(w.row_ptr_bytes) + align_up(w.col_idx_bytes);
  if (scratch_bytes != nullptr) *scratch_bytes = w.scratch_bytes;
  g_last_error.clear();
  return FP2_OK;
}

fp2_status fp2_pool(const fp2_problem* problem, const fp2_sparse_params* params, const fp2_pooled* pooled,
                    void* scratch, size_t scratch_bytes, fp2_stream_t stream) {
  Ctx c;
  fp2_status s;
  if ((s = validate(problem, params, c)) != FP2_OK) return s;
  if ((s = check_scratch(scratch, scratch_bytes, c.ws.scratch_bytes)) != FP2_OK) return s;
  if ((s = check_pooled(pooled, true, problem->dtype == FP2_E4M3)) != FP2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_status(scratch, st)) != FP2_OK) return s;
  if (c.T == 0) return FP2_OK;
  return run_pool(problem, params, c, pooled, scratch, st);
}

fp2_status fp2_discover(const fp2_problem* problem, const fp2_sparse_params* params, const fp2_pooled* pooled,
                        const fp2_index* index, void* scratch, size_t scratch_bytes, fp2_stream_t stream) {
  Ctx c;
  fp2_status s;
  if ((s = validate(problem, params, c)) != FP2_OK) return s;
  if ((s = check_scratch(scratch, scratch_bytes, c.ws.scratch_bytes)) != FP2_OK) return s;
  if ((s = check_pooled(pooled, true, false)) != FP2_OK) return s;
  if ((s = check_index(index, c)) != FP2_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_status(scratch, st)) != FP2_OK) return s;
  if (c.T == 0) return FP2_OK;
  return run_discover(problem, params, c, pooled, index, scratch, st);
}

fp2_status fp2_attend(const fp2_problem* problem, const fp2_sparse_params* params, const fp2_pooled* pooled,
                      const fp2_index* index, void* out, float* lse, void* scratch, size_t scratch_bytes,
                      fp2_stream_t stream) {
  Ctx c;
  fp2_status s;
  if ((s = validate(problem, params, c)) != FP2_OK) return s;
  if ((s = check_scratch(scratch, scratch_bytes, c.ws.scratch_bytes)) != FP2_OK) return s;
  if ((s = check_pooled(pooled, false, problem->dtype == FP2_E4M3)) != FP2_OK) return s;
  if ((s = check_index(index, c)) != FP2_OK) return s;
  if (out == nullptr || !aligned16(out)) return fail(FP2_ERR_INVALID_ARG, "out must be a 16-byte aligned pointer");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_status(scratch, st)) != FP2_OK) return s;
  if (c.T == 0) return FP2_OK;
  return run_attend(problem, params, c, pooled, index, out, lse, scratch, st);
}

fp2_status fp2_prefill(const fp2_problem* problem, const fp2_sparse_params* params, void* out, float* lse,
                       void* scratch, size_t scratch_bytes, fp2_stream_t stream) {
  Ctx c;
  fp2_status s;
  if ((s = validate(problem, params, c)) != FP2_OK) return s;
  if ((s = check_scratch(scratch, scratch_bytes, c.ws.prefill_scratch_bytes)) != FP2_OK) return s;
  if (out == nullptr || !aligned16(out)) return fail(FP2_ERR_INVALID_ARG, "out must be a 16-byte aligned pointer");
  char* base = static_cast<char*>(scratch);
  fp2_pooled pl{reinterpret_cast<float*>(base + c.off_qbar), reinterpret_cast<float*>(base + c.off_kbar),
                reinterpret_cast<float*>(base + c.off_vbar), base + c.off_kbm, base + c.off_vbm,
                c.ws.v16_bytes ? base + c.off_v16 : nullptr};
  fp2_index ix{reinterpret_cast<int32_t*>(base + c.off_rowptr), reinterpret_cast<int32_t*>(base + c.off_colidx),
               std::max<int64_t>(c.cap, 1)};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_status(scratch, st)) != FP2_OK) return s;
  if (c.T == 0) return FP2_OK;
  if ((s = run_pool(problem, params, c, &pl, scratch, st)) != FP2_OK) return s;
  if ((s = run_discover(problem, params, c, &pl, &ix, scratch, st)) != FP2_OK) return s;
  return run_attend(problem, params, c, &pl, &ix, out, lse, scratch, st);
}

fp2_status fp2_get_device_status(const void* scratch, uint32_t* status_out) {
  if (scratch == nullptr || status_out == nullptr) return fail(FP2_ERR_INVALID_ARG, "NULL argument");
  uint32_t w = 0;
  const cudaError_t e = cudaMemcpy(&w, scratch, sizeof(w), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  *status_out = w;
  if (w & FP2_DEV_TIMEOUT) return fail(FP2_ERR_TIMEOUT, "a device-side wait timed out");
  if (w & FP2_DEV_CHECK) return fail(FP2_ERR_CHECK_FAILED, "a device-side check of the checked build failed");
  if (w & (FP2_DEV_PAGE_OOB | FP2_DEV_INDEX_OOB | FP2_DEV_CAPACITY))
    return fail(FP2_ERR_DEVICE_BOUNDS, "device reported an out-of-range page id, index entry or capacity overflow");
  return FP2_OK;
}

fp2_status fp2_debug_set(int32_t key, int64_t value) {
  switch (key) {
    case FP2_DEBUG_WAIT_LIMIT_NS:
      if (value != 0 && (value < 100000 || value > 10000000000LL))
        return fail(FP2_ERR_INVALID_ARG, "wait limit must be 0 (default) or in [1e5, 1e10] ns");
      g_wait_limit_ns.store(value);
      return FP2_OK;
    case FP2_DEBUG_WITHHOLD_K_TILE:
      if (value < -1 || value > FP2_MAX_BLOCKS) return fail(FP2_ERR_INVALID_ARG, "tile must be -1 or in [0, FP2_MAX_BLOCKS]");
      g_withhold_k_tile.store(value);
      return FP2_OK;
    case FP2_DEBUG_MISCOUNT_LOAD:
      if (value < -1 || value > 2 * FP2_MAX_BLOCKS) return fail(FP2_ERR_INVALID_ARG, "load must be -1 or in [0, 2 * FP2_MAX_BLOCKS]");
      g_miscount_load.store(value);
      return FP2_OK;
    default:
      return fail(FP2_ERR_INVALID_ARG, "unknown debug key");
  }
}

const char* fp2_last_error(void) { return g_last_error.c_str(); }

int32_t fp2_version(void) { return 10000; }

uint32_t fp2_build_flags(void) {
#if defined(FP2_CHECKED) && FP2_CHECKED
  return FP2_BUILD_CHECKED;
#else
  return 0u;
#endif
}

}  // extern "C"
