// lf_api.cu — the C ABI of liblf (declared in include/lf.h): argument validation, launch
// configuration and tensor-map set-up for the four hierarchical-sparse-attention stages.
// The library is one translation unit: the kernels are included below.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <algorithm>
#include <cmath>
#include <mutex>
#include <string.h>

#include "lf_common.cuh"
#include "lf_select.cuh"
#include "lf_attn.cuh"
#include "lf_fused.cuh"
#include "lf_fp8.cuh"

using lf::Dims;

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Validates the plain sizes and derives the rest.  Returns LF_OK or an error code.
int make_dims(const lf_shape* s, Dims* D) {
  if (s == nullptr || D == nullptr) return LF_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return LF_ERR_UNSUPPORTED;
  if (s->block != 64 && s->block != 128) return LF_ERR_UNSUPPORTED;
  if (s->H < 1 || s->tokens_per_frame < 1 || s->n_cur_frames < 1 || s->n_hist < 0 ||
      s->n_sink < 0 || s->n_slots < 0)
    return LF_ERR_INVALID_ARG;
  if (s->tokens_per_frame > LF_MAX_T) return LF_ERR_UNSUPPORTED;
  if (s->n_hist + s->n_sink > LF_MAX_FRAMES) return LF_ERR_UNSUPPORTED;
  if ((s->n_hist > 0 || s->n_sink > 0) && s->n_slots < 1) return LF_ERR_INVALID_ARG;
  if (s->n_hist > 0 && (s->k_f < 1 || s->k_b < 1)) return LF_ERR_INVALID_ARG;
  if (s->k_c < 0) return LF_ERR_INVALID_ARG;
  if (!(s->scale > 0.f) || s->scale > 1e30f) return LF_ERR_INVALID_ARG;
  const long long ncur = (long long)s->n_cur_frames * s->tokens_per_frame;
  if (ncur > (1LL << 30) / ((long long)s->H * s->d)) return LF_ERR_UNSUPPORTED;
  if ((long long)s->n_slots * s->tokens_per_frame * s->H * s->d > (1LL << 40))
    return LF_ERR_UNSUPPORTED;
  Dims d{};
  d.H = s->H; d.d = s->d; d.T = s->tokens_per_frame; d.B = s->block;
  d.Fc = s->n_cur_frames; d.F = s->n_hist; d.S = s->n_sink; d.n_slots = s->n_slots;
  d.nbpf = lf::cdiv(d.T, d.B);
  d.nqb = d.Fc * d.nbpf;
  d.ncur = d.Fc * d.T;
  d.kf = d.F > 0 ? (s->k_f < d.F ? s->k_f : d.F) : 0;
  d.kb = d.F > 0 ? (s->k_b < d.nbpf ? s->k_b : d.nbpf) : 0;
  d.nsel = d.kf * d.kb;
  d.kc = s->k_c > 0 ? (s->k_c < d.nqb ? s->k_c : d.nqb) : 0;
  d.scale = s->scale;
  if (d.nsel > LF_MAX_SELECTED) return LF_ERR_UNSUPPORTED;
  if (d.kc > 0 && d.nqb > LF_MAX_CUR_BLOCKS) return LF_ERR_UNSUPPORTED;
  if (lf::plan_stride(d) > lf::kMaxPlan) return LF_ERR_UNSUPPORTED;
  *D = d;
  return LF_OK;
}

int check_slots(const int32_t* slots, int n, int n_slots) {
  if (n == 0) return LF_OK;
  if (slots == nullptr) return LF_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (slots[i] < 0 || slots[i] >= n_slots) return LF_ERR_INVALID_ARG;
  return LF_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LF_OK : LF_ERR_CUDA; }

constexpr size_t kMaxSmem = 227 * 1024;   // opt-in shared memory per block on sm_100
static_assert(LF_MAX_PLAN == lf::kMaxPlan, "the header's key-plan limit is the kernels'");

// --------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess && q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// bf16 rows of H*d channels: 2-D [rows, H*d] or 3-D [slots, T, H*d]; box = 64 channels x
// 64 rows (x 1 slot); 128-byte swizzle; out-of-bounds elements read as zero.
int encode_rows(CUtensorMap* m, const void* base, int HD, long long rows, int slots) {
  auto fn = encode_fn();
  if (fn == nullptr) return LF_ERR_CUDA;
  const cuuint32_t rank = slots > 0 ? 3 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)rows, (cuuint64_t)(slots > 0 ? slots : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)HD * 2, (cuuint64_t)HD * 2 * (cuuint64_t)rows};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LF_OK : LF_ERR_CUDA;
}

// e4m3 rows of H*d bytes: 2-D [rows, H*d] or 3-D [slots, T, H*d]; box = 128 bytes x 64 rows
// (x 1 slot) -- one 128-byte swizzled row per token at d = 128; out-of-bounds bytes read as
// zero.
int encode_rows_e4m3(CUtensorMap* m, const void* base, int HD, long long rows, int slots) {
  auto fn = encode_fn();
  if (fn == nullptr) return LF_ERR_CUDA;
  const cuuint32_t rank = slots > 0 ? 3 : 2;
  cuuint64_t dims[3] = {(cuuint64_t)HD, (cuuint64_t)rows, (cuuint64_t)(slots > 0 ? slots : 1)};
  cuuint64_t strides[2] = {(cuuint64_t)HD, (cuuint64_t)HD * (cuuint64_t)rows};
  cuuint32_t box[3] = {128, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? LF_OK : LF_ERR_CUDA;
}

// e4m3 operands of the FP8 attention variant (null pointer: the bf16 path).
struct F8Args {
  const void* q8;          // [ncur, H, d] e4m3 codes
  const float* q_scale;    // [ncur, H]
  const void* k_cur8;      // [ncur, H, d]
  const void* k_cache8;    // [n_slots, T, H, d]
  const float* k_scale;    // [H]
};

// ---------------------------------------------------------------- launches
// Pooling of the query blocks, the history key blocks (D.F frames) and, when kc_blk is
// given, the current chunk's key blocks; then (k_frm given) the history frame means.
int launch_compress(const Dims& D, const void* q, const void* k_cache, const int32_t* hist_slots,
                    float* q_blk, float* k_blk, float* k_frm, cudaStream_t st,
                    const void* k_cur = nullptr, float* kc_blk = nullptr) {
  lf::PoolArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  a.q_blk = q_blk;
  a.k_blk = k_blk;
  a.k_pool = nullptr;
  a.k_cur = static_cast<const __nv_bfloat16*>(k_cur);
  a.kc_blk = kc_blk;
  for (int f = 0; f < D.F; ++f) a.hist_slots[f] = hist_slots[f];
  const int units = D.nqb + D.F * D.nbpf + (kc_blk != nullptr ? D.nqb : 0);
  const int vecs = D.H * D.d / 8;
  dim3 grid(units, lf::cdiv(vecs, lf::kPoolCols));
  lf::pool_blocks_kernel<<<grid, lf::kPoolThreads, 0, st>>>(a, D);
  if (D.F > 0 && k_frm != nullptr)
    lf::pool_frames_kernel<<<dim3(D.F, D.H), D.d, 0, st>>>(k_blk, k_frm, D);
  return cuda_status(cudaGetLastError());
}

// Block means of the keys of cache slots `slots[0..n)` into the pooled-key cache
// k_pool [n_slots, H, nbpf, d] (the pooling kernel over history units only).
int launch_pool_frames(const Dims& D, const void* k_cache, const int32_t* slots, int n,
                       float* k_pool, cudaStream_t st) {
  if (n == 0) return LF_OK;
  Dims Dp = D;
  Dp.nqb = 0;
  Dp.F = n;
  lf::PoolArgs a{};
  a.k_cache = static_cast<const __nv_bfloat16*>(k_cache);
  a.k_pool = k_pool;
  for (int f = 0; f < n; ++f) a.hist_slots[f] = slots[f];
  dim3 grid(n * D.nbpf, lf::cdiv(D.H * D.d / 8, lf::kPoolCols));
  lf::pool_blocks_kernel<<<grid, lf::kPoolThreads, 0, st>>>(a, Dp);
  return cuda_status(cudaGetLastError());
}

int launch_select_frames(const Dims& D, const float* q_blk, const float* k_frm,
                         int32_t* frame_idx, float* frame_score, cudaStream_t st) {
  const size_t smem = ((size_t)D.F * (D.d + 4) + (size_t)lf::kSelWarps * D.d) * sizeof(float);
  if (smem > kMaxSmem) return LF_ERR_UNSUPPORTED;
  auto kern = D.d == 128 ? lf::select_frames_kernel<128> : lf::select_frames_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return LF_ERR_CUDA;
  dim3 grid(lf::cdiv(D.nqb, lf::kSelWarps), D.H);
  kern<<<grid, lf::kSelWarps * 32, smem, st>>>(q_blk, k_frm, frame_idx, frame_score, D);
  return cuda_status(cudaGetLastError());
}

// Current-chunk block choice: own block plus the kc - 1 best others, per (head, query block).
int launch_select_current(const Dims& D, const float* q_blk, const float* kc_blk,
                          int32_t* cur_idx, cudaStream_t st) {
  const size_t smem = ((size_t)D.nqb * (D.d + 4) + (size_t)lf::kSelWarps * D.d) * sizeof(float);
  if (smem > kMaxSmem) return LF_ERR_UNSUPPORTED;
  auto kern = D.d == 128 ? lf::select_current_kernel<128> : lf::select_current_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return LF_ERR_CUDA;
  dim3 grid(lf::cdiv(D.nqb, lf::kSelWarps), D.H);
  kern<<<grid, lf::kSelWarps * 32, smem, st>>>(q_blk, kc_blk, cur_idx, D);
  return cuda_status(cudaGetLastError());
}

int launch_select_blocks(const Dims& D, const float* q_blk, const float* k_blk,
                         const int32_t* frame_idx, int32_t* block_idx, float* block_score,
                         cudaStream_t st) {
  const size_t smem = ((size_t)D.nbpf * (D.d + 4) + (size_t)lf::kSelBatch * D.d) * sizeof(float) +
                      (size_t)D.nqb * (1 + D.kf) * sizeof(int);
  if (smem > kMaxSmem) return LF_ERR_UNSUPPORTED;
  auto kern = D.d == 128 ? lf::select_blocks_kernel<128> : lf::select_blocks_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return LF_ERR_CUDA;
  kern<<<dim3(D.F, D.H, lf::kSelSplit), lf::kSelWarps * 32, smem, st>>>(
      q_blk, k_blk, frame_idx, block_idx, block_score, D);
  return cuda_status(cudaGetLastError());
}

// SM count of the current device (work decomposition and workspace sizing).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

// Work decomposition of the attention grid: full waves of whole tiles; if the last wave
// would be less than half full, its tiles are split into `pieces` key ranges each.
struct Split {
  int n_whole, n_tail, pieces;
};

// Test hooks set by lf_debug_configure (process-wide; defaults: 2 s wait limit, no stall,
// tail split allowed).
uint64_t g_dbg_wait_limit_ns = lf::kWaitLimitNs;
int g_dbg_stall = 0;
int g_dbg_tail_split = 1;

Split make_split(const Dims& D, int n_sm) {
  const int ntot = lf::tile_count(D) * D.H;
  Split sp{ntot, 0, 1};
  if (n_sm <= 0 || !g_dbg_tail_split) return sp;
  const int R = ntot % n_sm;
  if (R == 0 || 2 * R > n_sm) return sp;
  int p = n_sm / R;
  p = p < lf::kMaxPieces ? p : lf::kMaxPieces;
  const int n_min = lf::min_key_tiles(D);        // every tile has at least this many
  p = p < n_min ? p : n_min;
  if (p < 2) return sp;
  sp.n_whole = ntot - R;
  sp.n_tail = R;
  sp.pieces = p;
  return sp;
}

struct AttnWs {
  uint32_t* plan;
  int32_t* plan_cnt;
  float* part_o;
  float* part_ml;
  size_t bytes;
};

// plan | counts | partial O of up to n_sm pieces | their (m, l)
AttnWs carve_attn(const Dims& D, void* base, int n_sm) {
  AttnWs w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t n) { uint8_t* r = p ? p + off : nullptr; off += align_up(n, 256); return r; };
  const size_t nt = (size_t)lf::tile_count(D) * D.H;
  const size_t units = n_sm > 0 ? (size_t)n_sm : 0;
  w.plan = reinterpret_cast<uint32_t*>(take(nt * lf::plan_stride(D) * sizeof(uint32_t)));
  w.plan_cnt = reinterpret_cast<int32_t*>(take(nt * sizeof(int32_t)));
  w.part_o = reinterpret_cast<float*>(take(units * 128 * D.d * sizeof(float)));
  w.part_ml = reinterpret_cast<float*>(take(units * 2 * 128 * sizeof(float)));
  w.bytes = off;
  return w;
}

size_t attn_ws_bytes(const Dims& D) { return carve_attn(D, nullptr, sm_count()).bytes; }

template <int HD, int BLK, bool F8 = false>
int launch_attn_t(const Dims& D, lf::AttnParams& p, int grid, cudaStream_t st) {
  using L = lf::AttnLayout<HD>;
  auto kern = lf::attn_kernel<HD, BLK, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return LF_ERR_CUDA;
  // the in-kernel register split assumes the launch register count; never launch otherwise
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, kern) != cudaSuccess) return LF_ERR_CUDA;
  if (fa.numRegs != lf::kLaunchRegs) return LF_ERR_UNSUPPORTED;
  kern<<<grid, lf::kAttnThreads, L::kAlloc, st>>>(p, D);
  return cuda_status(cudaGetLastError());
}

int launch_attn(const Dims& D, const void* q, const void* k_cur, const void* v_cur,
                const void* k_cache, const void* v_cache, const int32_t* hist_slots,
                const int32_t* sink_slots, const int32_t* block_idx, const int32_t* cur_idx,
                void* out, float* lse, void* workspace, cudaStream_t st,
                bool plans_ready = false, const F8Args* f8 = nullptr) {
  const int n_sm = sm_count();
  if (n_sm <= 0) return LF_ERR_CUDA;
  const AttnWs w = carve_attn(D, workspace, n_sm);
  // key plans (unless the fused selection already wrote them)
  if (!plans_ready)
    lf::plan_kernel<<<dim3(lf::cdiv(lf::tile_count(D), lf::kPlanWarps), D.H), lf::kPlanWarps * 32, 0, st>>>(
        D.F > 0 ? block_idx : nullptr, D.kc > 0 ? cur_idx : nullptr, w.plan, w.plan_cnt, D);
  const Split sp = make_split(D, n_sm);
  int rc = cuda_status(cudaGetLastError());
  if (rc != LF_OK) return rc;

  lf::AttnParams p;
  memset(&p, 0, sizeof(p));
  const int HD = D.H * D.d;
  if (f8 != nullptr) {                 // e4m3 queries and keys, bf16 values
    if ((rc = encode_rows_e4m3(&p.tm_q, f8->q8, HD, D.ncur, 0)) != LF_OK) return rc;
    if ((rc = encode_rows_e4m3(&p.tm_kc, f8->k_cur8, HD, D.ncur, 0)) != LF_OK) return rc;
    p.q_scale = f8->q_scale;
    p.k_scale = f8->k_scale;
  } else {
    if ((rc = encode_rows(&p.tm_q, q, HD, D.ncur, 0)) != LF_OK) return rc;
    if ((rc = encode_rows(&p.tm_kc, k_cur, HD, D.ncur, 0)) != LF_OK) return rc;
  }
  if ((rc = encode_rows(&p.tm_vc, v_cur, HD, D.ncur, 0)) != LF_OK) return rc;
  if (D.F + D.S > 0) {
    if (f8 != nullptr)
      rc = encode_rows_e4m3(&p.tm_kh, f8->k_cache8, HD, D.T, D.n_slots);
    else
      rc = encode_rows(&p.tm_kh, k_cache, HD, D.T, D.n_slots);
    if (rc != LF_OK) return rc;
    if ((rc = encode_rows(&p.tm_vh, v_cache, HD, D.T, D.n_slots)) != LF_OK) return rc;
  } else {   // no cache frames: the maps are never used; point them at the current chunk
    p.tm_kh = p.tm_kc;
    p.tm_vh = p.tm_vc;
  }
  p.plan = w.plan;
  p.plan_cnt = w.plan_cnt;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.tiles_per_head = lf::tile_count(D);
  p.n_whole = sp.n_whole;
  p.pieces = sp.pieces;
  p.part_o = w.part_o;
  p.part_ml = w.part_ml;
  p.wait_limit_ns = g_dbg_wait_limit_ns;
  p.debug_stall = g_dbg_stall;
  for (int i = 0; i < D.S; ++i) p.slots[i] = sink_slots[i];
  for (int i = 0; i < D.F; ++i) p.slots[D.S + i] = hist_slots[i];
  const int grid = sp.n_whole + sp.n_tail * sp.pieces;
  if (f8 != nullptr)
    rc = D.B == 64 ? launch_attn_t<128, 64, true>(D, p, grid, st)
                   : launch_attn_t<128, 128, true>(D, p, grid, st);
  else if (D.d == 128)
    rc = D.B == 64 ? launch_attn_t<128, 64>(D, p, grid, st) : launch_attn_t<128, 128>(D, p, grid, st);
  else
    rc = D.B == 64 ? launch_attn_t<64, 64>(D, p, grid, st) : launch_attn_t<64, 128>(D, p, grid, st);
  if (rc != LF_OK || sp.n_tail == 0) return rc;
  lf::merge_kernel<<<dim3(sp.n_tail, 128 / lf::kMergeRows), 256, 0, st>>>(p, D, D.d);
  return cuda_status(cudaGetLastError());
}

// forward workspace carve-up
struct FwdWs {
  float *q_blk, *k_blk, *k_frm, *scores, *kc_blk;
  int32_t *frame_idx, *block_idx, *cur_idx;
  void* attn;
  size_t bytes;
};

FwdWs carve(const Dims& D, void* base) {
  FwdWs w{};
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t n) { uint8_t* r = p ? p + off : nullptr; off += align_up(n, 256); return r; };
  w.q_blk = reinterpret_cast<float*>(take((size_t)D.H * D.nqb * D.d * 4));
  w.k_blk = reinterpret_cast<float*>(take((size_t)D.H * D.F * D.nbpf * D.d * 4));
  w.k_frm = reinterpret_cast<float*>(take((size_t)D.H * D.F * D.d * 4));
  w.scores = reinterpret_cast<float*>(take((size_t)D.H * D.nqb * D.F * D.nbpf * 4));
  w.frame_idx = reinterpret_cast<int32_t*>(take((size_t)D.H * D.nqb * D.kf * 4));
  w.block_idx = reinterpret_cast<int32_t*>(take((size_t)D.H * D.nqb * D.nsel * 4));
  w.kc_blk = reinterpret_cast<float*>(take((size_t)D.H * (D.kc > 0 ? D.nqb : 0) * D.d * 4));
  w.cur_idx = reinterpret_cast<int32_t*>(take((size_t)D.H * D.nqb * D.kc * 4));
  w.attn = take(attn_ws_bytes(D));
  w.bytes = off;
  return w;
}

// Block scores (from the per-call pooled keys w.k_blk, or from the pooled-key cache k_pool
// through hist_slots) and the pick kernel (frame and block top-k, key plans).
// Scores of every history block against every pooled query block into sa.scores.
int launch_block_scores(const Dims& D, const lf::ScoreArgs& sa, cudaStream_t stream) {
  const dim3 grid(lf::cdiv(D.F * D.nbpf, lf::kScoreRows), D.H, lf::cdiv(D.nqb, lf::kScoreQb));
  auto kern = D.d == 128 ? lf::block_scores_kernel<128> : lf::block_scores_kernel<64>;
  const size_t smem = D.d == 128 ? lf::score_smem<128>() : lf::score_smem<64>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return LF_ERR_CUDA;
  kern<<<grid, lf::kScoreThreads, smem, stream>>>(sa, D);
  return cuda_status(cudaGetLastError());
}

int launch_scores_pick(const Dims& D, const FwdWs& w, const float* k_pool,
                       const int32_t* hist_slots, const AttnWs& aw, int32_t* bidx,
                       cudaStream_t stream) {
  lf::ScoreArgs sa{};
  sa.q_blk = w.q_blk;
  sa.k_blk = w.k_blk;
  sa.k_pool = k_pool;
  sa.scores = w.scores;
  if (k_pool != nullptr)
    for (int f = 0; f < D.F; ++f) sa.slots[f] = hist_slots[f];
  int rc = launch_block_scores(D, sa, stream);
  if (rc != LF_OK) return rc;
  const size_t smem = lf::fused_select_smem(D);
  if (cudaFuncSetAttribute(lf::select_pick_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return LF_ERR_CUDA;
  // with a sparse current chunk the key plans also hold current blocks: plan_kernel
  // builds them, the pick kernel writes the lists only
  lf::select_pick_kernel<<<dim3(lf::cdiv(D.nqb, lf::kFuseQb), D.H), lf::kPickThreads, smem,
                           stream>>>(w.scores, bidx, D.kc > 0 ? nullptr : aw.plan, aw.plan_cnt, D);
  return cuda_status(cudaGetLastError());
}

// Stages (a)-(c) into `bidx`: pooling, then the fused selection (which also writes the
// attention key plans into the workspace, *plans_ready) when the shape allows it, else the
// separate frame-pooling, frame-selection and block-selection kernels.
int run_select(const Dims& D, const void* q, const void* k_cache, const int32_t* hist_slots,
               const FwdWs& w, int32_t* bidx, cudaStream_t stream, bool* plans_ready,
               const void* k_cur = nullptr) {
  int rc;
  *plans_ready = false;
  float* kc_blk = k_cur != nullptr ? w.kc_blk : nullptr;   // also pool the current keys
  if (lf::fused_select_ok(D) && lf::fused_select_smem(D) <= kMaxSmem) {
    if ((rc = launch_compress(D, q, k_cache, hist_slots, w.q_blk, w.k_blk, nullptr, stream,
                              k_cur, kc_blk)) != LF_OK)
      return rc;
    const int n_sm = sm_count();
    if (n_sm <= 0) return LF_ERR_CUDA;
    const AttnWs aw = carve_attn(D, w.attn, n_sm);
    if ((rc = launch_scores_pick(D, w, nullptr, hist_slots, aw, bidx, stream)) != LF_OK) return rc;
    *plans_ready = D.kc == 0;
    return LF_OK;
  }
  if ((rc = launch_compress(D, q, k_cache, hist_slots, w.q_blk, w.k_blk, w.k_frm, stream,
                            k_cur, kc_blk)) != LF_OK)
    return rc;
  if ((rc = launch_select_frames(D, w.q_blk, w.k_frm, w.frame_idx, nullptr, stream)) != LF_OK)
    return rc;
  return launch_select_blocks(D, w.q_blk, w.k_blk, w.frame_idx, bidx, nullptr, stream);
}

// Current-chunk selection: pooling of the query and current key blocks (one launch),
// then the own block plus the kc - 1 best others per (head, query block).
int run_select_current(const Dims& D, const void* q, const void* k_cur, const FwdWs& w,
                       int32_t* cur_idx, cudaStream_t stream) {
  Dims Dq = D;
  Dq.F = 0;                                      // no history units in this pooling launch
  int rc = launch_compress(Dq, q, nullptr, nullptr, w.q_blk, nullptr, nullptr, stream, k_cur,
                           w.kc_blk);
  if (rc != LF_OK) return rc;
  return launch_select_current(D, w.q_blk, w.kc_blk, cur_idx, stream);
}

// ---------------------------------------------------------------- fixed scratch
// Scratch for lf_block_sparse_attn_noalloc: a fixed-size array in device global memory.
// It exists on a device once this library's module is loaded there (with lazy module
// loading, at the first use of the library on that device) and lives until the context
// is destroyed.  Host code must not use the symbol itself as a device address: the address
// is looked up with cudaGetSymbolAddress, with the device current, and cached together
// with the context it belongs to, so that a context re-created after cudaDeviceReset (the
// module reloaded, possibly at another address) gets a fresh lookup.
constexpr size_t kNoAllocScratchBytes = 16u << 20;       // 16 MiB
static __device__ __align__(256) uint8_t g_lf_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
struct ScratchAddr {
  CUcontext ctx;
  void* addr;
};
ScratchAddr g_noalloc_addr[kMaxDevices] = {};

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
std::once_flag g_ctx_once;

// The current context of the calling thread (the runtime's primary context once any
// runtime call has initialised the device), or null if it cannot be read.
CUcontext current_context() {
  std::call_once(g_ctx_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  });
  CUcontext c = nullptr;
  if (g_ctx_current == nullptr || g_ctx_current(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the fixed scratch on the current device and context (looked up on
// the first call in that context).
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LF_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  ScratchAddr& e = g_noalloc_addr[dev];
  const CUcontext ctx = current_context();       // null before the runtime's first use
  if (ctx == nullptr || e.addr == nullptr || e.ctx != ctx) {
    void* p = nullptr;
    // the lookup itself makes the device's primary context current
    if (cudaGetSymbolAddress(&p, g_lf_noalloc_scratch) != cudaSuccess || p == nullptr)
      return LF_ERR_CUDA;
    const CUcontext now = current_context();
    if (now == nullptr) return LF_ERR_CUDA;
    e.ctx = now;
    e.addr = p;
  }
  *out = e.addr;
  return LF_OK;
}

}  // namespace

// ===================================================================== C ABI
extern "C" {

int lf_cag_schedule(int32_t n_chunks, int32_t first, float mean_sparsity, float final_sparsity,
                    const int32_t* n_hist, int32_t n_bpf, int32_t kf_max, float* keep,
                    int32_t* k_f, int32_t* k_b) {
  const bool budgets = n_hist != nullptr || k_f != nullptr || k_b != nullptr;
  if (n_chunks < 1 || n_chunks > 4096 || first < 1 || first > n_chunks || keep == nullptr ||
      n_bpf < 1 || kf_max < 1 || !(mean_sparsity >= 0.f && mean_sparsity < 1.f) ||
      !(final_sparsity >= 0.f && final_sparsity < 1.f) ||
      (budgets && (n_hist == nullptr || k_f == nullptr || k_b == nullptr)))
    return LF_ERR_INVALID_ARG;
  // mean over the sparse chunks of alpha_i = 1/sqrt(i), and alpha of the last chunk
  double a_mean = 0.0;
  for (int i = first; i <= n_chunks; ++i) a_mean += 1.0 / std::sqrt((double)i);
  a_mean /= (double)(n_chunks - first + 1);
  const double a_last = 1.0 / std::sqrt((double)n_chunks);
  double beta = 0.0, s_base = final_sparsity;
  if (first < n_chunks) {
    // s_base - beta * a_mean = mean, s_base - beta * a_last = final
    beta = ((double)final_sparsity - (double)mean_sparsity) / (a_mean - a_last);
    s_base = (double)final_sparsity + beta * a_last;
  } else if (std::fabs((double)mean_sparsity - (double)final_sparsity) > 1e-6) {
    return LF_ERR_INVALID_ARG;
  }
  for (int i = 1; i <= n_chunks; ++i) {
    double r = 1.0;
    if (i >= first) r = std::min(1.0, std::max(0.0, 1.0 - (s_base - beta / std::sqrt((double)i))));
    keep[i - 1] = (float)r;
    if (!budgets) continue;
    const int F = n_hist[i - 1];
    if (F <= 0) {
      k_f[i - 1] = k_b[i - 1] = 0;
    } else if (i < first) {
      k_f[i - 1] = F;
      k_b[i - 1] = n_bpf;
    } else {
      const int kf = std::min(kf_max, F);
      // halves round up; the 1e-9 keeps an exact half that arrives as x.4999999 from
      // rounding in the keep ratio on the upper side
      const int kb = (int)std::floor(r * F * n_bpf / kf + 0.5 + 1e-9);
      k_f[i - 1] = kf;
      k_b[i - 1] = std::min(n_bpf, std::max(1, kb));
    }
  }
  return LF_OK;
}

int lf_abi_version(void) { return LF_ABI_VERSION; }

const char* lf_status_string(int s) {
  switch (s) {
    case LF_OK: return "ok";
    case LF_ERR_INVALID_ARG: return "invalid argument";
    case LF_ERR_UNSUPPORTED: return "unsupported shape";
    case LF_ERR_CUDA: return "CUDA error";
    case LF_ERR_TIMEOUT: return "device wait timed out";
    case LF_ERR_WORKSPACE: return "workspace missing or too small";
    case LF_ERR_BAD_INDEX: return "index out of range in a device list";
    default: return "unknown status";
  }
}

int lf_compress(const lf_shape* shape, const void* q, const void* k_cache,
                const int32_t* hist_slots, float* q_blk, float* k_blk, float* k_frm,
                cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (q == nullptr || q_blk == nullptr || !aligned(q, 16) || !aligned(q_blk, 16))
    return LF_ERR_INVALID_ARG;
  if (D.F > 0) {
    if (k_cache == nullptr || k_blk == nullptr || k_frm == nullptr || !aligned(k_cache, 16) ||
        !aligned(k_blk, 16) || !aligned(k_frm, 16))
      return LF_ERR_INVALID_ARG;
    if ((rc = check_slots(hist_slots, D.F, D.n_slots)) != LF_OK) return rc;
  }
  return launch_compress(D, q, k_cache, hist_slots, q_blk, k_blk, k_frm, stream);
}

int lf_select_frames(const lf_shape* shape, const float* q_blk, const float* k_frm,
                     int32_t* frame_idx, float* frame_score, cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.F < 1) return LF_ERR_INVALID_ARG;
  if (q_blk == nullptr || k_frm == nullptr || frame_idx == nullptr || !aligned(q_blk, 16) ||
      !aligned(k_frm, 16) || !aligned(frame_idx, 4) || (frame_score && !aligned(frame_score, 4)))
    return LF_ERR_INVALID_ARG;
  return launch_select_frames(D, q_blk, k_frm, frame_idx, frame_score, stream);
}

int lf_select_blocks(const lf_shape* shape, const float* q_blk, const float* k_blk,
                     const int32_t* frame_idx, int32_t* block_idx, float* block_score,
                     cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.F < 1) return LF_ERR_INVALID_ARG;
  if (q_blk == nullptr || k_blk == nullptr || frame_idx == nullptr || block_idx == nullptr ||
      !aligned(q_blk, 16) || !aligned(k_blk, 16) || !aligned(frame_idx, 4) ||
      !aligned(block_idx, 4) || (block_score && !aligned(block_score, 4)))
    return LF_ERR_INVALID_ARG;
  return launch_select_blocks(D, q_blk, k_blk, frame_idx, block_idx, block_score, stream);
}

size_t lf_attn_workspace_size(const lf_shape* shape) {
  Dims D;
  if (make_dims(shape, &D) != LF_OK) return 0;
  return attn_ws_bytes(D);
}

int lf_block_sparse_attn(const lf_shape* shape, const void* q, const void* k_cur,
                         const void* v_cur, const void* k_cache, const void* v_cache,
                         const int32_t* hist_slots, const int32_t* sink_slots,
                         const int32_t* block_idx, const int32_t* cur_idx, void* out,
                         float* lse, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (q == nullptr || k_cur == nullptr || v_cur == nullptr || out == nullptr ||
      !aligned(q, 16) || !aligned(k_cur, 16) || !aligned(v_cur, 16) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)))
    return LF_ERR_INVALID_ARG;
  if (D.F + D.S > 0 && (k_cache == nullptr || v_cache == nullptr || !aligned(k_cache, 16) ||
                        !aligned(v_cache, 16)))
    return LF_ERR_INVALID_ARG;
  if (D.F > 0 && (block_idx == nullptr || !aligned(block_idx, 4))) return LF_ERR_INVALID_ARG;
  if (D.kc > 0 && (cur_idx == nullptr || !aligned(cur_idx, 4))) return LF_ERR_INVALID_ARG;
  if ((rc = check_slots(hist_slots, D.F, D.n_slots)) != LF_OK) return rc;
  if ((rc = check_slots(sink_slots, D.S, D.n_slots)) != LF_OK) return rc;
  const size_t need = attn_ws_bytes(D);
  if (need == 0) return LF_ERR_CUDA;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need)
    return LF_ERR_WORKSPACE;
  return launch_attn(D, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots, block_idx,
                     cur_idx, out, lse, workspace, stream);
}

int lf_block_sparse_attn_e4m3(const lf_shape* shape, const void* q8, const float* q_scale,
                              const void* k_cur8, const void* v_cur, const void* k_cache8,
                              const void* v_cache, const float* k_scale,
                              const int32_t* hist_slots, const int32_t* sink_slots,
                              const int32_t* block_idx, const int32_t* cur_idx, void* out,
                              float* lse, void* workspace, size_t workspace_bytes,
                              cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.d != 128) return LF_ERR_UNSUPPORTED;
  if (q8 == nullptr || q_scale == nullptr || k_cur8 == nullptr || v_cur == nullptr ||
      k_scale == nullptr || out == nullptr || !aligned(q8, 16) || !aligned(k_cur8, 16) ||
      !aligned(v_cur, 16) || !aligned(out, 16) || !aligned(q_scale, 4) ||
      !aligned(k_scale, 4) || (lse && !aligned(lse, 4)))
    return LF_ERR_INVALID_ARG;
  if (D.F + D.S > 0 && (k_cache8 == nullptr || v_cache == nullptr || !aligned(k_cache8, 16) ||
                        !aligned(v_cache, 16)))
    return LF_ERR_INVALID_ARG;
  if (D.F > 0 && (block_idx == nullptr || !aligned(block_idx, 4))) return LF_ERR_INVALID_ARG;
  if (D.kc > 0 && (cur_idx == nullptr || !aligned(cur_idx, 4))) return LF_ERR_INVALID_ARG;
  if ((rc = check_slots(hist_slots, D.F, D.n_slots)) != LF_OK) return rc;
  if ((rc = check_slots(sink_slots, D.S, D.n_slots)) != LF_OK) return rc;
  const size_t need = attn_ws_bytes(D);
  if (need == 0) return LF_ERR_CUDA;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need)
    return LF_ERR_WORKSPACE;
  const F8Args f8{q8, q_scale, k_cur8, k_cache8, k_scale};
  return launch_attn(D, nullptr, nullptr, v_cur, nullptr, v_cache, hist_slots, sink_slots,
                     block_idx, cur_idx, out, lse, workspace, stream, false, &f8);
}

int lf_quantize_e4m3(const void* x, int64_t rows, int32_t H, int32_t d, const float* head_scale,
                     uint8_t* x8, float* row_scale, cudaStream_t stream) {
  if (rows < 0 || H < 1 || (d != 64 && d != 128)) return LF_ERR_INVALID_ARG;
  if (rows > ((int64_t)1 << 40) / ((int64_t)H * d)) return LF_ERR_UNSUPPORTED;
  if (rows == 0) return LF_OK;
  if (x == nullptr || x8 == nullptr || !aligned(x, 16) || !aligned(x8, 16) ||
      (head_scale == nullptr && (row_scale == nullptr || !aligned(row_scale, 4))) ||
      (head_scale != nullptr && !aligned(head_scale, 4)))
    return LF_ERR_INVALID_ARG;
  const long long threads = rows * H * (d / 8);   // d / 8 threads per (row, head)
  const int block = 256;
  lf::quantize_e4m3_kernel<<<(unsigned)((threads + block - 1) / block), block, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), rows, H, d, head_scale, x8, row_scale);
  return cuda_status(cudaGetLastError());
}

int lf_e4m3_head_scales(const void* const* xs, const int64_t* rows, int32_t n, int32_t H,
                        int32_t d, float* head_scale, cudaStream_t stream) {
  if (n < 1 || n > 16 || xs == nullptr || rows == nullptr || H < 1 || (d != 64 && d != 128) ||
      head_scale == nullptr || !aligned(head_scale, 4))
    return LF_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i)
    if (rows[i] < 0 || (rows[i] > 0 && (xs[i] == nullptr || !aligned(xs[i], 16))))
      return LF_ERR_INVALID_ARG;
  // head_scale first holds the amax bit patterns, then (in place) the scales
  if (cudaMemsetAsync(head_scale, 0, (size_t)H * sizeof(float), stream) != cudaSuccess)
    return LF_ERR_CUDA;
  unsigned int* bits = reinterpret_cast<unsigned int*>(head_scale);
  for (int i = 0; i < n; ++i) {
    if (rows[i] == 0) continue;
    const long long blocks = std::min<long long>((rows[i] + 255) / 256, 1024);
    lf::head_amax_kernel<<<dim3((unsigned)blocks, H), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(xs[i]), rows[i], H, d, bits);
  }
  lf::head_scale_kernel<<<(H + 127) / 128, 128, 0, stream>>>(bits, H, head_scale);
  return cuda_status(cudaGetLastError());
}

size_t lf_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int lf_block_sparse_attn_noalloc(const lf_shape* shape, const void* q, const void* k_cur,
                                 const void* v_cur, const void* k_cache, const void* v_cache,
                                 const int32_t* hist_slots, const int32_t* sink_slots,
                                 const int32_t* block_idx, void* out, float* lse,
                                 cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.kc > 0) return LF_ERR_INVALID_ARG;                     // takes no current-chunk list
  const size_t need = attn_ws_bytes(D);
  if (need == 0) return LF_ERR_CUDA;
  if (need > kNoAllocScratchBytes) return LF_ERR_WORKSPACE;   // shape needs more scratch
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch)) != LF_OK) return rc;
  return lf_block_sparse_attn(shape, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots,
                              block_idx, nullptr, out, lse, scratch, kNoAllocScratchBytes,
                              stream);
}

size_t lf_forward_workspace_size(const lf_shape* shape) {
  Dims D;
  if (make_dims(shape, &D) != LF_OK) return 0;
  return carve(D, nullptr).bytes;
}

int lf_forward_chunk(const lf_shape* shape, const void* q, const void* k_cur,
                     const void* v_cur, const void* k_cache, const void* v_cache,
                     const int32_t* hist_slots, const int32_t* sink_slots,
                     void* workspace, size_t workspace_bytes, void* out, float* lse,
                     int32_t* block_idx_out, int32_t* cur_idx_out, cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (q == nullptr || k_cur == nullptr || v_cur == nullptr || out == nullptr ||
      !aligned(q, 16) || !aligned(k_cur, 16) || !aligned(v_cur, 16) || !aligned(out, 16) ||
      (lse && !aligned(lse, 4)) || (block_idx_out && !aligned(block_idx_out, 4)) ||
      (cur_idx_out && !aligned(cur_idx_out, 4)))
    return LF_ERR_INVALID_ARG;
  if (D.F + D.S > 0 && (k_cache == nullptr || v_cache == nullptr || !aligned(k_cache, 16) ||
                        !aligned(v_cache, 16)))
    return LF_ERR_INVALID_ARG;
  if ((rc = check_slots(hist_slots, D.F, D.n_slots)) != LF_OK) return rc;
  if ((rc = check_slots(sink_slots, D.S, D.n_slots)) != LF_OK) return rc;
  const FwdWs need = carve(D, nullptr);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need.bytes)
    return LF_ERR_WORKSPACE;
  const FwdWs w = carve(D, workspace);
  int32_t* bidx = block_idx_out ? block_idx_out : w.block_idx;
  int32_t* cidx = cur_idx_out ? cur_idx_out : w.cur_idx;
  bool plans_ready = false;
  if (D.F > 0) {
    // with a sparse current chunk the same pooling launch also pools the current keys
    if ((rc = run_select(D, q, k_cache, hist_slots, w, bidx, stream, &plans_ready,
                         D.kc > 0 ? k_cur : nullptr)) != LF_OK)
      return rc;
    if (D.kc > 0 && (rc = launch_select_current(D, w.q_blk, w.kc_blk, cidx, stream)) != LF_OK)
      return rc;
  } else if (D.kc > 0) {
    if ((rc = run_select_current(D, q, k_cur, w, cidx, stream)) != LF_OK) return rc;
  }
  return launch_attn(D, q, k_cur, v_cur, k_cache, v_cache, hist_slots, sink_slots, bidx, cidx,
                     out, lse, w.attn, stream, plans_ready);
}

int lf_select_current(const lf_shape* shape, const void* q, const void* k_cur,
                      int32_t* cur_idx, void* workspace, size_t workspace_bytes,
                      cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.kc < 1) return LF_ERR_INVALID_ARG;
  if (q == nullptr || k_cur == nullptr || cur_idx == nullptr || !aligned(q, 16) ||
      !aligned(k_cur, 16) || !aligned(cur_idx, 4))
    return LF_ERR_INVALID_ARG;
  const FwdWs need = carve(D, nullptr);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need.bytes)
    return LF_ERR_WORKSPACE;
  return run_select_current(D, q, k_cur, carve(D, workspace), cur_idx, stream);
}

size_t lf_select_workspace_size(const lf_shape* shape) { return lf_forward_workspace_size(shape); }

int lf_select_chunk(const lf_shape* shape, const void* q, const void* k_cache,
                    const int32_t* hist_slots, int32_t* block_idx, void* workspace,
                    size_t workspace_bytes, cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.F < 1) return LF_ERR_INVALID_ARG;
  if (q == nullptr || k_cache == nullptr || block_idx == nullptr || !aligned(q, 16) ||
      !aligned(k_cache, 16) || !aligned(block_idx, 4))
    return LF_ERR_INVALID_ARG;
  if ((rc = check_slots(hist_slots, D.F, D.n_slots)) != LF_OK) return rc;
  const FwdWs need = carve(D, nullptr);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need.bytes)
    return LF_ERR_WORKSPACE;
  bool plans_ready = false;
  return run_select(D, q, k_cache, hist_slots, carve(D, workspace), block_idx, stream, &plans_ready);
}

int lf_select_chunk_1d(const lf_shape* shape, const void* q, const void* k_cache,
                       const int32_t* hist_slots, int32_t* block_idx, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.F < 1) return LF_ERR_INVALID_ARG;
  if (q == nullptr || k_cache == nullptr || block_idx == nullptr || !aligned(q, 16) ||
      !aligned(k_cache, 16) || !aligned(block_idx, 4))
    return LF_ERR_INVALID_ARG;
  if ((rc = check_slots(hist_slots, D.F, D.n_slots)) != LF_OK) return rc;
  const int nb = D.F * D.nbpf;
  if (nb > lf::kFuseMaxBlocks) return LF_ERR_UNSUPPORTED;
  const FwdWs need = carve(D, nullptr);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need.bytes)
    return LF_ERR_WORKSPACE;
  const FwdWs w = carve(D, workspace);
  if ((rc = launch_compress(D, q, k_cache, hist_slots, w.q_blk, w.k_blk, nullptr, stream)) != LF_OK)
    return rc;
  lf::ScoreArgs sa{};
  sa.q_blk = w.q_blk;
  sa.k_blk = w.k_blk;
  sa.k_pool = nullptr;
  sa.scores = w.scores;
  if ((rc = launch_block_scores(D, sa, stream)) != LF_OK) return rc;
  int n2 = 2;
  while (n2 < nb) n2 <<= 1;
  const size_t smem = (size_t)n2 * 3 * 4;
  lf::select_topk_kernel<<<dim3(D.nqb, D.H), lf::kTopkThreads, smem, stream>>>(
      w.scores, block_idx, D, n2);
  return cuda_status(cudaGetLastError());
}

size_t lf_pooled_cache_bytes(const lf_shape* shape) {
  Dims D;
  if (make_dims(shape, &D) != LF_OK) return 0;
  return (size_t)D.n_slots * D.H * D.nbpf * D.d * sizeof(float);
}

int lf_pool_frames(const lf_shape* shape, const void* k_cache, const int32_t* slots,
                   int32_t n, float* k_pool, cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (n < 0 || n > LF_MAX_FRAMES) return LF_ERR_INVALID_ARG;
  if (n == 0) return LF_OK;
  if (k_cache == nullptr || k_pool == nullptr || !aligned(k_cache, 16) || !aligned(k_pool, 16))
    return LF_ERR_INVALID_ARG;
  if ((rc = check_slots(slots, n, D.n_slots)) != LF_OK) return rc;
  return launch_pool_frames(D, k_cache, slots, n, k_pool, stream);
}

int lf_select_chunk_cached(const lf_shape* shape, const void* q, const float* k_pool,
                           const int32_t* hist_slots, int32_t* block_idx, void* workspace,
                           size_t workspace_bytes, cudaStream_t stream) {
  Dims D;
  int rc = make_dims(shape, &D);
  if (rc != LF_OK) return rc;
  if (D.F < 1) return LF_ERR_INVALID_ARG;
  if (q == nullptr || k_pool == nullptr || block_idx == nullptr || !aligned(q, 16) ||
      !aligned(k_pool, 16) || !aligned(block_idx, 4))
    return LF_ERR_INVALID_ARG;
  if ((rc = check_slots(hist_slots, D.F, D.n_slots)) != LF_OK) return rc;
  if (!lf::fused_select_ok(D) || lf::fused_select_smem(D) > kMaxSmem) return LF_ERR_UNSUPPORTED;
  const FwdWs need = carve(D, nullptr);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need.bytes)
    return LF_ERR_WORKSPACE;
  const FwdWs w = carve(D, workspace);
  Dims Dq = D;
  Dq.F = 0;                                  // pool the query blocks only
  if ((rc = launch_compress(Dq, q, nullptr, hist_slots, w.q_blk, nullptr, nullptr, stream)) != LF_OK)
    return rc;
  const int n_sm = sm_count();
  if (n_sm <= 0) return LF_ERR_CUDA;
  return launch_scores_pick(D, w, k_pool, hist_slots, carve_attn(D, w.attn, n_sm), block_idx,
                            stream);
}

int lf_debug_configure(uint64_t wait_limit_ns, int stall, int tail_split) {
  if (wait_limit_ns > 10ull * lf::kWaitLimitNs) return LF_ERR_INVALID_ARG;
  g_dbg_wait_limit_ns = wait_limit_ns == 0 ? lf::kWaitLimitNs : wait_limit_ns;
  g_dbg_stall = stall != 0;
  g_dbg_tail_split = tail_split != 0;
  return LF_OK;
}

#ifdef LF_TRACE
int lf_debug_set_trace(void* buf, void* cta_buf) {
  unsigned long long* p = static_cast<unsigned long long*>(buf);
  unsigned long long* q = static_cast<unsigned long long*>(cta_buf);
  if (cudaMemcpyToSymbol(lf::g_lf_trace, &p, sizeof(p)) != cudaSuccess) return LF_ERR_CUDA;
  return cudaMemcpyToSymbol(lf::g_lf_cta_trace, &q, sizeof(q)) == cudaSuccess ? LF_OK : LF_ERR_CUDA;
}
#endif

int lf_device_status(int reset) {
  int v = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return LF_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&v, lf::g_lf_status, sizeof(int)) != cudaSuccess) return LF_ERR_CUDA;
  if (reset && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(lf::g_lf_status, &zero, sizeof(int)) != cudaSuccess) return LF_ERR_CUDA;
  }
  return v;
}

}  // extern "C"
