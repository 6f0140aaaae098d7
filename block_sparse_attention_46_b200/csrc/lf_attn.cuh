// lf_attn.cuh — stage (d) of hierarchical sparse attention: block-sparse attention of the
// current chunk's queries over (current chunk, dense) + (sink frames, dense) + (the
// history blocks each query block selected), one joint softmax per query.
//
// [LF-gist 2.2] "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
// Attention" (gist.science explainer), section 2.2, execution step: attention is computed
// only on the selected frame-block pairs.  [LF-yly 三] the youleyou article, section 三:
// the two selection stages give a block-level mask consumed by a sparse attention kernel.
// [RF 三] Rolling Forcing article, section 三: sink frames are kept as global anchors.
//
// sm_100a design (one CTA = one head x one 128-row query tile):
//   * a query tile is two 64-token query blocks (block 64) or one 128-token block
//     (block 128); a key tile is 128 keys: 128 contiguous current-chunk tokens, or two
//     64-token blocks (one 128-token block) taken from the tile's key plan;
//   * the key plan of a tile (sink blocks, then the sorted union of its query blocks'
//     selected blocks, each with a bit per query block that selected it) is built by
//     plan_kernel; a key column a row's query block did not select is masked to -inf;
//   * Q, then K and V tiles, stream with TMA (128-byte swizzle, zero fill out of bounds)
//     into one ring of 160 KB (five 32 KB stages at d = 128) in the order the MMAs consume
//     them, the K tiles issued by warp 0 and the V tiles by warp 2; warp 1 issues the
//     tcgen05.mma S = Q K^T into one of two tensor-memory buffers (S of tile l+1 is computed
//     while the softmax works on tile l) and warp 3, once it has staged the tile's key plan
//     into shared memory, the PVs: O_w += P_w V_w over softmax warpgroup w's 64 keys;
//   * warps 4-11 are two softmax warpgroups; warpgroup w takes keys [64w, 64w + 64) of
//     every key tile and keeps its own fp32 online softmax state and O_w over them, one
//     query row per thread (the row's tensor-memory lane): S from tensor memory, P as bf16
//     pairs written over S, O_w rescaled in tensor memory only when its row maximum grows
//     by more than 2^8 (lazy rescale); the two states are merged in the epilogue;
//   * every mbarrier wait is bounded; on expiry the CTA drains and returns with
//     LF_ERR_TIMEOUT recorded.
#pragma once
#include <cuda.h>
#include "lf_common.cuh"

namespace lf {

constexpr int kMaxPlan = 2048;          // key-plan entries per query tile
constexpr int kAttnThreads = 384;

// Plan entry: bits 0-1 = which of the tile's two query blocks selected it (bit 0: rows
// 0-63 or the single 128-row block; bit 1: rows 64-127), bits 4-15 = block in frame,
// bits 16-27 = frame position: sinks [0, S), history frames [S, S + F), and, when the
// current chunk is sparse, the current chunk's frames [S + F, S + F + F_c).
__host__ __device__ inline uint32_t plan_pack(int p, int b, uint32_t mask) {
  return ((uint32_t)p << 16) | ((uint32_t)b << 4) | mask;
}

__host__ __device__ inline int tile_count(const Dims& D) {
  return D.B == 64 ? cdiv(D.nqb, 2) : D.nqb;
}
__host__ __device__ inline int plan_stride(const Dims& D) {
  return D.S * D.nbpf + (D.B == 64 ? 2 : 1) * (D.kc + D.nsel);
}
// Key tiles every query tile has at least: the dense current chunk, or the key blocks of
// one query block's lists (sinks, kept current blocks, selected history blocks).
__host__ __device__ inline int min_key_tiles(const Dims& D) {
  const int per = D.B == 64 ? 2 : 1;
  return (D.kc > 0 ? 0 : cdiv(D.ncur, 128)) + cdiv(D.S * D.nbpf + D.kc + D.nsel, per);
}

// ---------------------------------------------------------------------------------
// Key plan of each (query tile, head): one warp.  Sink blocks first (selected by both
// query blocks), then the sorted union of the two ascending block lists; the position
// of an element in the union is its rank in its own list plus the number of smaller
// elements of the other list minus the common elements counted twice.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ int lower_bound_s(const int32_t* a, int n, int v) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (a[mid] < v) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// One warp writes the sorted union of a tile's two ascending id lists A and B (shared
// memory, already validated; nB = 0 when the tile has one query block) at out[0..), each
// id as the plan entry of frame position p_base + id / nbpf, block id % nbpf, with a bit
// per list holding it.  The position of an element in the union is its rank in its own
// list plus the number of smaller elements of the other list minus the common elements
// counted twice.  Returns the entry count.
__device__ __forceinline__ int warp_write_union(const int32_t* sa, int nA, const int32_t* sb,
                                                int nB, uint32_t* out, int p_base, int nbpf) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  int carry = 0;
  for (int i0 = 0; i0 < nA; i0 += 32) {
    const int i = i0 + lane;
    const bool valid = i < nA;
    const int a = valid ? sa[i] : 0x7fffffff;
    const int cb = lower_bound_s(sb, nB, a);
    const bool inB = valid && cb < nB && sb[cb] == a;
    const uint32_t bal = __ballot_sync(0xffffffffu, inB);
    if (valid) {
      const int pos = i + cb - (carry + __popc(bal & lt));
      out[pos] = plan_pack(p_base + a / nbpf, a % nbpf, inB ? 3u : 1u);
    }
    carry += __popc(bal);
  }
  const int ncommon = carry;
  carry = 0;
  for (int j0 = 0; j0 < nB; j0 += 32) {
    const int j = j0 + lane;
    const bool valid = j < nB;
    const int b = valid ? sb[j] : 0x7fffffff;
    const int ca = lower_bound_s(sa, nA, b);
    const bool inA = valid && ca < nA && sa[ca] == b;
    const uint32_t bal = __ballot_sync(0xffffffffu, inA);
    if (valid && !inA) {
      const int pos = j + ca - (carry + __popc(bal & lt));
      out[pos] = plan_pack(p_base + b / nbpf, b % nbpf, 2u);
    }
    carry += __popc(bal);
  }
  return nA + nB - ncommon;
}

// Stages one query tile's two ascending lists of n ids each (B absent when qbB < 0) from
// `lists` [H, nqb, n] into shared memory and checks them (ids in [0, lim), strictly
// ascending).  Returns false, for the whole warp, if either list is invalid.
__device__ __forceinline__ bool warp_stage_lists(const int32_t* lists, int n, int lim, int h,
                                                 int qa, int qbB, const Dims& D, int32_t* sa,
                                                 int32_t* sb) {
  const int lane = threadIdx.x & 31;
  stage_words(sa, lists + ((size_t)h * D.nqb + qa) * n, n, lane, 32);
  if (qbB >= 0) stage_words(sb, lists + ((size_t)h * D.nqb + qbB) * n, n, lane, 32);
  __syncwarp();
  const int nB = qbB >= 0 ? n : 0;
  bool bad = false;
  for (int i = lane; i < n; i += 32) bad |= sa[i] < 0 || sa[i] >= lim || (i > 0 && sa[i - 1] >= sa[i]);
  for (int i = lane; i < nB; i += 32) bad |= sb[i] < 0 || sb[i] >= lim || (i > 0 && sb[i - 1] >= sb[i]);
  return !__any_sync(0xffffffffu, bad);
}

constexpr int kPlanWarps = 4;

// Key plan of each (query tile, head), one warp: sink blocks (kept by both query blocks),
// then the union of the query blocks' current-chunk lists (when the current chunk is
// sparse), then the union of their history lists.  A list that fails validation is
// dropped and LF_ERR_BAD_INDEX recorded.
__global__ void __launch_bounds__(kPlanWarps * 32)
plan_kernel(const int32_t* __restrict__ block_idx, const int32_t* __restrict__ cur_idx,
            uint32_t* __restrict__ plan, int32_t* __restrict__ plan_cnt, const Dims D) {
  __shared__ int32_t s_ab[kPlanWarps][2][LF_MAX_SELECTED];
  const int ntiles = tile_count(D);
  const int t = blockIdx.x * kPlanWarps + (threadIdx.x >> 5), h = blockIdx.y;
  const int lane = threadIdx.x & 31;
  if (t >= ntiles) return;
  int32_t* sa = s_ab[threadIdx.x >> 5][0];
  int32_t* sb = s_ab[threadIdx.x >> 5][1];
  uint32_t* out = plan + ((size_t)h * ntiles + t) * plan_stride(D);
  const int qa = D.B == 64 ? 2 * t : t;
  const int qbB = (D.B == 64 && 2 * t + 1 < D.nqb) ? 2 * t + 1 : -1;
  const int nsink = D.S * D.nbpf;
  for (int e = lane; e < nsink; e += 32) out[e] = plan_pack(e / D.nbpf, e % D.nbpf, 3u);
  int cnt = nsink;
  bool bad = false;
  if (D.kc > 0) {
    if (warp_stage_lists(cur_idx, D.kc, D.nqb, h, qa, qbB, D, sa, sb))
      cnt += warp_write_union(sa, D.kc, sb, qbB >= 0 ? D.kc : 0, out + cnt, D.S + D.F, D.nbpf);
    else
      bad = true;
    __syncwarp();
  }
  if (D.F > 0 && D.nsel > 0 && block_idx != nullptr) {
    if (warp_stage_lists(block_idx, D.nsel, D.F * D.nbpf, h, qa, qbB, D, sa, sb))
      cnt += warp_write_union(sa, D.nsel, sb, qbB >= 0 ? D.nsel : 0, out + cnt, D.S, D.nbpf);
    else
      bad = true;
  }
  if (lane == 0) {
    if (bad) record_status(LF_ERR_BAD_INDEX);
    plan_cnt[(size_t)h * ntiles + t] = cnt;
  }
}


// ---------------------------------------------------------------------------------
// Attention kernel
// ---------------------------------------------------------------------------------
struct AttnParams {
  CUtensorMap tm_q;    // [ncur, H*d] bf16, box 64 x 64
  CUtensorMap tm_kc;   // current-chunk keys, same geometry
  CUtensorMap tm_vc;
  CUtensorMap tm_kh;   // cache keys [n_slots, T, H*d], box 1 x 64 x 64
  CUtensorMap tm_vh;
  const uint32_t* plan;
  const int32_t* plan_cnt;
  __nv_bfloat16* out;  // [ncur, H, d]
  float* lse;          // [H, ncur] or null
  // work decomposition: CTAs [0, n_whole) take tiles whole; the remaining tiles (the last
  // partial wave) are split into `pieces` key ranges each, written as partial softmax
  // states to part_o / part_ml and combined by merge_kernel
  int tiles_per_head;
  int n_whole;
  int pieces;
  float* part_o;       // [n_tail * pieces, 128, d] unnormalised O
  float* part_ml;      // [n_tail * pieces, 2, 128] row max (log2 units) and row sum
  const float* q_scale;       // e4m3 variant: [ncur, H] query scales (tm_q and tm_kc/tm_kh
  const float* k_scale;       // then map e4m3 Q and K), [H] key scales; else unused
  uint64_t wait_limit_ns;     // limit of every bounded wait of the launch (kWaitLimitNs)
  int debug_stall;     // test hook: when set, CTA 0 never arms its Q barrier, so its
                       // first wait runs out (the timeout and drain path)
  int slots[LF_MAX_FRAMES];   // cache slot of frame position p (sinks, then history)
};

// barrier indices: ring full/empty barriers follow these
// PV barriers: kBarPVDone + buffer, completion of both PVs of a tile
// kBarDone: completion of everything the two MMA threads issued (one arrival each)
enum BarId { kBarQ = 0, kBarSFull = 1, kBarDone = 3, kBarPVDone = 4, kBarRing = 6 };
// named barriers (0 is __syncthreads): the epilogue's exchange, the producers' drain, and
// per softmax warpgroup w the hand-off of each tile's P to the PV thread's warp.  Both
// sides wait (bar.sync) once per tile, so no warp can arrive for a later tile before a
// tile's hand-off is complete, also when an aborted wait has desynchronised the loops.
constexpr int kNbEpilogue = 1, kNbProducers = 2, kNbP = 3;   // kNbP + w
constexpr int kNbPThreads = 160;                              // 4 softmax warps + PV warp

template <int HD>
struct AttnLayout {
  static constexpr int NH = HD / 64;                 // 64-column halves of the head dim
  static constexpr int kRegion = 128 * 128;          // bytes of one 128-row x 64-col half
  static constexpr int kQ = 0;
  static constexpr int kQBytes = NH * kRegion;
  // one ring of K and V tiles in the order the MMAs consume them: K0, K1, V0, K2, V1, ...
  static constexpr int kSlots = HD == 128 ? 5 : 10;
  static constexpr int kRing = kQ + kQBytes;
  static constexpr int kStageBytes = NH * kRegion;
  static constexpr int kPlan = kRing + kSlots * kStageBytes;
  static constexpr int kRed = kPlan + kMaxPlan * 4;  // per-row (m, l) of both warpgroups
  static constexpr int kBar = kRed + 2 * 2 * 128 * 4;
  static constexpr int kNumBars = 2 * kSlots + kBarRing;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;       // slack for 1024-byte alignment
  // tensor-memory columns: two O accumulators (one per softmax warpgroup), two S buffers;
  // warpgroup w's P (bf16 pairs) overwrites columns [64w, 64w + 32) of the S buffer it was
  // computed from
  static constexpr uint32_t kColO0 = 0, kColO1 = 128, kColS0 = 256, kColS1 = 384,
                            kTmemCols = 512;
};

// position of a tile in the ring's load order: K0, K1, V0, K2, V1, K3, V2, ...
__device__ __forceinline__ int ring_pos_k(int j) { return j < 2 ? j : 2 * j - 1; }
__device__ __forceinline__ int ring_pos_v(int i) { return 2 + 2 * i; }
// inverse: the tile at ring position q (K_j when isK, else V_j)
__device__ __forceinline__ int ring_tile(int q, bool& isK) {
  if (q < 2) { isK = true; return q; }
  if ((q & 1) == 0) { isK = false; return (q - 2) >> 1; }
  isK = true;
  return (q + 1) >> 1;
}

// Maximum of N (64 or 128) values: eight independent chains of three-input max.
template <int N>
__device__ __forceinline__ float row_max(const float* v) {
  float m[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmax3f(v[k], v[8 + k], v[16 + k]);
#pragma unroll
  for (int i = 24; i < N - 8; i += 16)
#pragma unroll
    for (int k = 0; k < 8; ++k) m[k] = fmax3f(m[k], v[i + k], v[i + 8 + k]);
#pragma unroll
  for (int k = 0; k < 8; ++k) m[k] = fmaxf(m[k], v[N - 8 + k]);
  return fmaxf(fmax3f(m[0], m[1], m[2]), fmax3f(fmax3f(m[3], m[4], m[5]), m[6], m[7]));
}

constexpr int kSoftmaxWarps = 8;          // two warpgroups, one 64-key half of every tile each
// Register split: launched at 168 per thread (384 threads); the load/MMA warpgroup gives
// registers to the two softmax warpgroups: 128 x 72 + 256 x 216 <= 384 x 168.
constexpr int kLaunchRegs = 168, kLowRegs = 72, kHighRegs = 216;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kAttnThreads * kLaunchRegs, "register split");

// F8: queries and keys are e4m3 codes (one byte per element, 128-byte rows at d = 128, one
// swizzled region per 128-row tile), S = Q K^T by tcgen05.mma kind::f8f6f4 (exact products,
// fp32 accumulation) and the scales enter the softmax's per-row factor; V, P and the PV
// MMAs are as in the bf16 path.
template <int HD, int BLK, bool F8 = false>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const __grid_constant__ AttnParams P, const Dims D) {
  static_assert(!F8 || HD == 128, "the e4m3 path has d = 128");
  using L = AttnLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* s_plan = reinterpret_cast<uint32_t*>(smem + L::kPlan);
  float* s_red = reinterpret_cast<float*>(smem + L::kRed);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
  volatile int* s_stop = reinterpret_cast<volatile int*>(smem + L::kMisc + 8);   // producers' ends

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work unit: a whole tile, or piece k of a tail tile
  int pos, piece = -1, tail = 0;
  if ((int)blockIdx.x < P.n_whole) {
    pos = blockIdx.x;
  } else {
    tail = (blockIdx.x - P.n_whole) / P.pieces;
    piece = (blockIdx.x - P.n_whole) % P.pieces;
    pos = P.n_whole + tail;
  }
  // tiles in index order (head-major): the CTAs running at any time read the history of
  // a few heads, which stays in L2; the last partial wave is split (see n_whole)
  const int tile = pos;
  const int h = tile / P.tiles_per_head, t = tile % P.tiles_per_head;

  // query blocks of this tile
  const int qbA = BLK == 64 ? 2 * t : t;
  const int qbB = (BLK == 64 && 2 * t + 1 < D.nqb) ? 2 * t + 1 : -1;
  const int tokA = (qbA / D.nbpf) * D.T + (qbA % D.nbpf) * BLK;
  const int tokB = qbB >= 0 ? (qbB / D.nbpf) * D.T + (qbB % D.nbpf) * BLK : D.ncur;

  const int cnt = P.plan_cnt[tile];
  const int n_dense = D.kc > 0 ? 0 : cdiv(D.ncur, 128);   // sparse current chunk: in the plan
  const int n_sparse = BLK == 64 ? cdiv(cnt, 2) : cnt;
  const int n_tile = n_dense + n_sparse;
  // this CTA's key tiles: [j0, j0 + n_iter); local index l = j - j0 drives the pipeline
  int j0 = 0, n_iter = n_tile;
  if (piece >= 0) {
    j0 = (int)((long long)piece * n_tile / P.pieces);
    n_iter = (int)((long long)(piece + 1) * n_tile / P.pieces) - j0;
  }

  // TMA loads of Q, and of ring position q (tile l, a key tile when isK) armed on its slot's
  // full barrier; sparse tiles read the staged key plan, dense ones (j < n_dense) do not
  auto load_q = [&]() {
    if (F8) {
      mbar_arrive_expect_tx(&bars[kBarQ], 128 * HD);         // e4m3: one byte per element
      uint8_t* dst = smem + L::kQ;
      tma_load_2d(dst, &P.tm_q, &bars[kBarQ], h * HD, tokA);
      tma_load_2d(dst + 64 * 128, &P.tm_q, &bars[kBarQ], h * HD, BLK == 64 ? tokB : tokA + 64);
    } else {
      mbar_arrive_expect_tx(&bars[kBarQ], L::kQBytes);
      for (int c = 0; c < L::NH; ++c) {
        uint8_t* dst = smem + L::kQ + c * L::kRegion;
        tma_load_2d(dst, &P.tm_q, &bars[kBarQ], h * HD + c * 64, tokA);
        tma_load_2d(dst + 64 * 128, &P.tm_q, &bars[kBarQ], h * HD + c * 64,
                    BLK == 64 ? tokB : tokA + 64);
      }
    }
  };
  auto load_pos = [&](int q, bool isK, int l) {
    uint64_t* full = &bars[kBarRing];
    const int slot = q % L::kSlots;
    const int j = j0 + l;
    LF_TR(isK ? 0 : 1, l);
    const bool f8 = F8 && isK;                     // an e4m3 key tile: one 16 KB region
    const int nreg = f8 ? 1 : L::NH;
    const int xcol = f8 ? h * HD : 0;               // x coordinate base: bytes / elements
    mbar_arrive_expect_tx(&full[slot], f8 ? 128 * HD : L::kStageBytes);
    uint8_t* st = smem + L::kRing + slot * L::kStageBytes;
    const CUtensorMap* tm_cur = isK ? &P.tm_kc : &P.tm_vc;
    const CUtensorMap* tm_hist = isK ? &P.tm_kh : &P.tm_vh;
    for (int box = 0; box < 2; ++box) {
      if (j < n_dense) {
        const int row = j * 128 + box * 64;
        for (int c = 0; c < nreg; ++c)
          tma_load_2d(st + c * L::kRegion + box * 64 * 128, tm_cur, &full[slot],
                      f8 ? xcol : h * HD + c * 64, row);
      } else {
        const int u = j - n_dense;
        int slot_id = 0, tok = 0;
        int p = -1;                                    // -1: padding past the plan's end
        const int e = BLK == 64 ? 2 * u + box : u;
        if (e < cnt) {
          const uint32_t pe = s_plan[e];
          p = (int)(pe >> 16);
          tok = (int)((pe >> 4) & 0xFFFu) * BLK + (BLK == 64 ? 0 : box * 64);
          if (p < D.S + D.F) slot_id = P.slots[p];
        }
        if (p < 0 || p >= D.S + D.F) {
          // a block of the current chunk (2-D map), or padding: rows from ncur on are
          // out of bounds and read as zero (the columns are masked anyway)
          const int row = p < 0 ? D.ncur : (p - D.S - D.F) * D.T + tok;
          for (int c = 0; c < nreg; ++c)
            tma_load_2d(st + c * L::kRegion + box * 64 * 128, tm_cur, &full[slot],
                        f8 ? xcol : h * HD + c * 64, row);
        } else {
          for (int c = 0; c < nreg; ++c)
            tma_load_3d(st + c * L::kRegion + box * 64 * 128, tm_hist, &full[slot],
                        f8 ? xcol : h * HD + c * 64, tok, slot_id);
        }
      }
    }
  };
  int pre = 0;                                     // ring positions loaded in the set-up
  if (threadIdx.x == 0) {
    mbar_init(&bars[kBarQ], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kBarSFull + s], 1);
    }
    for (int q = 0; q < 2 * L::kSlots; ++q) mbar_init(&bars[kBarRing + q], 1);
    mbar_init(&bars[kBarDone], 2);
    mbar_init(&bars[kBarPVDone], 1);
    mbar_init(&bars[kBarPVDone + 1], 1);
    *s_abort = 0;
    fence_mbar_init();
    // Q and the first key tiles when they are dense (no key plan needed) go out now, so
    // their latency overlaps the tensor-memory allocation and the plan staging
    prefetch_tmap(&P.tm_q); prefetch_tmap(&P.tm_kc); prefetch_tmap(&P.tm_kh);
    prefetch_tmap(&P.tm_vc); prefetch_tmap(&P.tm_vh);
    if (!(P.debug_stall && blockIdx.x == 0)) load_q();
    for (; pre < 2 && pre < n_iter && j0 + pre < n_dense; ++pre) load_pos(pre, true, pre);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, L::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    LF_TR_CTA(0, smid());
    LF_TR_CTA(1, globaltimer_ns());
    LF_TR_CTA(3, n_iter);
  }
  if (warp == 3) stage_words(s_plan, P.plan + (size_t)tile * plan_stride(D), cnt, lane, 32);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp < 4) {
  regs_dec<kLowRegs>();
  // -------------------------------------------------------------- producers
  // Two threads issue the loads: warp 0 the K tiles, warp 2 the V tiles, each in ring order
  // within its own positions (a single thread issuing both cannot keep the ring filled
  // ahead of the MMAs on gathered key blocks).
  if (warp == 0 || warp == 2) {
    uint64_t* full = &bars[kBarRing];
    uint64_t* empty = &bars[kBarRing + L::kSlots];
    const int n_pos = 2 * n_iter + 1;               // V of the last tile sits at 2n
    const bool kside = warp == 0;
    if (lane == 0) {
      int q = kside ? pre : 2;                      // K positions below pre went in the set-up
      for (; q < n_pos; ++q) {
        bool isK;
        const int l = ring_tile(q, isK);
        if (isK != kside || (isK && l >= n_iter)) continue;   // the other side's, or no load
        const int slot = q % L::kSlots;
        const int rnd = q / L::kSlots;
        if (rnd > 0 && !mbar_wait(&empty[slot], (rnd & 1) ^ 1, s_abort, P.wait_limit_ns)) break;
        load_pos(q, isK, l);
      }
      s_stop[kside ? 0 : 1] = q;                    // positions of this side below q issued
    }
    __syncwarp();
    named_bar_sync(kNbProducers, 64);
    // drain: every load issued must land before the CTA may exit.  A load whose slot was
    // issued again (position + kSlots) is known to have landed; the others are waited for.
    if (warp == 0 && lane == 0) {
      const int qk = s_stop[0], qv = s_stop[1];
      auto issued = [&](int x) {
        if (x >= n_pos) return false;
        bool isK;
        const int lx = ring_tile(x, isK);
        if (isK && lx >= n_iter) return false;
        return x < (isK ? qk : qv);
      };
      for (int x = max(0, min(qk, qv) - 2 * L::kSlots); x < max(qk, qv); ++x)
        if (issued(x) && !issued(x + L::kSlots))
          mbar_wait_drain(&full[x % L::kSlots], (x / L::kSlots) & 1, P.wait_limit_ns);
    }
  }
  // -------------------------------------------------------------- MMA issuers
  // Two threads issue tcgen05.mma: warp 1 S_l = Q K_l^T into S buffer l & 1, warp 3 the PVs
  // of tile l (O_w += P_w V_w, warpgroup w's 64 keys) as soon as each warpgroup's P is
  // written.  S_{l+2} overwrites P_l, so it is issued only after both PVs of tile l have
  // completed (PV barrier of the buffer); the PV thread is never held up behind S MMAs.
  else if (warp == 1 || warp == 3) {
    constexpr uint32_t idesc_qk = F8 ? idesc_e4m3_f32(128, 128) : idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, HD, 0, 1);
    const uint32_t q_base = smem_u32(smem + L::kQ);
    const uint32_t ring_base = smem_u32(smem + L::kRing);
    uint64_t* full = &bars[kBarRing];
    uint64_t* empty = &bars[kBarRing + L::kSlots];
    bool ok = true;
    if (warp == 1 && lane == 0) {
      ok = mbar_wait(&bars[kBarQ], 0, s_abort, P.wait_limit_ns);
      for (int l = 0; ok && l < n_iter; ++l) {
        const int s = l & 1;
        const int q = ring_pos_k(l), slot = q % L::kSlots;
        LF_TR(2, l);
        // K_l (which lands early), then P_{l-2} (over this buffer) consumed: the PVs of tile
        // l-2 completed, the wait the issue depends on
        ok = mbar_wait(&full[slot], (q / L::kSlots) & 1, s_abort, P.wait_limit_ns);
        if (ok && l >= 2) ok = mbar_wait(&bars[kBarPVDone + s], ((l >> 1) & 1) ^ 1, s_abort, P.wait_limit_ns);
        if (!ok) break;
        LF_TR(3, l);
        tc_fence_after();
        const uint32_t d_tmem = tmem + (s ? L::kColS1 : L::kColS0);
        const uint32_t k_addr = ring_base + slot * L::kStageBytes;
        if constexpr (F8) {
#pragma unroll
          for (int ks = 0; ks < HD / 32; ++ks)          // 32 e4m3 elements = 32 bytes per MMA
            mma_e4m3_ss(d_tmem, smem_desc_sw128(q_base + ks * 32, 16, 1024),
                        smem_desc_sw128(k_addr + ks * 32, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
        } else {
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks) {
            const uint32_t off = (ks >> 2) * L::kRegion + (ks & 3) * 32;
            mma_bf16_ss(d_tmem, smem_desc_sw128(q_base + off, 16, 1024),
                        smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
          }
        }
        mma_commit(&bars[kBarSFull + s]);
        mma_commit(&empty[slot]);
      }
    } else if (warp == 3) {
      // every iteration meets both warpgroups at their barriers, also after a failed wait,
      // so that the syncs on each named barrier stay paired
      for (int l = 0; l < n_iter; ++l) {
        const int s = l & 1;
        const int qv = ring_pos_v(l), vslot = qv % L::kSlots;
        if (lane == 0 && ok) ok = mbar_wait(&full[vslot], (qv / L::kSlots) & 1, s_abort, P.wait_limit_ns);
        if (lane == 0) LF_TR(4, l);
        const uint32_t p_tmem = tmem + (s ? L::kColS1 : L::kColS0);
        for (int wg = 0; wg < 2; ++wg) {
          __syncwarp();
          named_bar_sync(kNbP + wg, kNbPThreads);            // P_l of warpgroup wg written
          if (lane == 0 && ok) {
            if (wg == 0) LF_TR(5, l);
            tc_fence_after();
            const uint32_t o_tmem = tmem + (wg ? L::kColO1 : L::kColO0);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {        // 16 keys per MMA, 8 P columns each
              const int ks = wg * 4 + k4;           // 16-key step within the V tile
              mma_bf16_ts(o_tmem, p_tmem + wg * 64 + k4 * 8,
                          smem_desc_sw128(ring_base + vslot * L::kStageBytes + ks * 16 * 128,
                                          L::kRegion, 1024),
                          idesc_pv, (l > 0 || k4 > 0) ? 1u : 0u);
            }
          }
        }
        if (lane == 0 && ok) {
          mma_commit(&bars[kBarPVDone + s]);
          mma_commit(&empty[vslot]);
        }
      }
    }
    // completion of everything this thread issued: epilogue may read O, tensor memory may
    // be freed once both threads' arrivals are in
    if (lane == 0) mma_commit(&bars[kBarDone]);
  }
  } else {
  regs_inc<kHighRegs>();
  // -------------------------------------------------------------- softmax + epilogue
  {
    const int wg = (warp - 4) >> 2;                        // keys [64 wg, 64 wg + 64) of each tile
    const int r = (threadIdx.x - 128) & 127;               // query row = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t row_bit = (BLK == 64 && r >= 64) ? 2u : 1u;
    const uint32_t o_col = wg ? L::kColO1 : L::kColO0;
    // scale * log2(e), times the row's query scale and the head's key scale for e4m3 Q/K
    float c = D.scale * 1.4426950408889634f;
    if constexpr (F8) {
      const int qb = BLK == 64 ? (r < 64 ? qbA : qbB) : qbA, i = BLK == 64 ? (r & 63) : r;
      const bool valid = qb >= 0 && i < block_len(D, qb % D.nbpf);
      const int tok = valid ? (qb / D.nbpf) * D.T + (qb % D.nbpf) * BLK + i : 0;
      c *= (valid ? P.q_scale[(size_t)tok * D.H + h] : 1.0f) * P.k_scale[h];
    }
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int l = 0; l < n_iter; ++l) {
      const int j = j0 + l, sb = l & 1;
      const uint32_t s_col = (sb ? L::kColS1 : L::kColS0) + wg * 64;
      if (threadIdx.x == 128) LF_TR(6, l);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull + sb], (l >> 1) & 1, s_abort, P.wait_limit_ns)) && ok;
      if (threadIdx.x == 128) LF_TR(7, l);
      tc_fence_after();
      float sv[64];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) tmem_ld32(t_row + s_col + ch * 32, sv + ch * 32);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) reg_fence32(sv + ch * 32);
      if (threadIdx.x == 128) LF_TR(8, l);

      // valid key columns [0, v) of this warpgroup's 64 (warp-uniform: a warp's 32 rows
      // belong to one query block)
      int v;
      if (j < n_dense) {
        v = max(0, min(64, D.ncur - j * 128 - wg * 64));
      } else {
        const int u = j - n_dense;
        if (BLK == 64) {
          const int e = 2 * u + wg;
          v = 0;
          if (e < cnt) {
            const uint32_t pe = s_plan[e];
            if (pe & row_bit) v = block_len(D, (pe >> 4) & 0xFFF);
          }
        } else {
          const uint32_t pe = s_plan[u];
          const int len = (pe & row_bit) ? block_len(D, (pe >> 4) & 0xFFF) : 0;
          v = max(0, min(64, len - wg * 64));
        }
      }
      // row maximum over the valid columns: a wholly valid half needs no masking, a wholly
      // masked one is left out (and skips its exponentials below); only a partly valid half
      // (a short last block of a frame, or the end of the current chunk) is masked
      float m_raw;
      if (v == 64) {
        m_raw = row_max<64>(sv);
      } else if (v > 0) {
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= v) sv[i] = -INFINITY;
        m_raw = row_max<64>(sv);
      } else {
        m_raw = -INFINITY;
      }
      const float m_tile = m_raw * c;
      float m_new = m_run;
      bool resc = false;
      if (m_tile > m_run + 8.0f) { m_new = m_tile; resc = true; }
      // lazy rescale of this group's O, once its last PV (PV_{l-1}) has completed
      if (l > 0 && __any_sync(0xffffffffu, resc)) {
        const bool w = mbar_wait(&bars[kBarPVDone + (sb ^ 1)], ((l - 1) >> 1) & 1, s_abort,
                                 P.wait_limit_ns);
        ok = __all_sync(0xffffffffu, w) && ok;
        tc_fence_after();
        const float a = resc ? exp2f(m_run - m_new) : 1.f;
#pragma unroll
        for (int ch = 0; ch < HD / 32; ++ch) {
          float o[32];
          tmem_ld32(t_row + o_col + ch * 32, o);
          tmem_ld_wait();
          reg_fence32(o);
#pragma unroll
          for (int q = 0; q < 32; ++q) o[q] *= a;
          tmem_st32(t_row + o_col + ch * 32, o);
        }
        if (resc) l_run *= a;
      }
      if (threadIdx.x == 128) LF_TR(9, l);
      const float mref = (m_new == -INFINITY) ? 0.f : m_new;
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-mref, -mref);
      float2 ps0 = make_float2(0.f, 0.f), ps1 = make_float2(0.f, 0.f);
      // probabilities in chunks of 32 keys packed to bf16 pairs and stored to tensor memory
      // (16 columns) at once; with no valid key for this row (warp-uniform) the chunk is
      // written as zeros without exponentials
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float pk[16];
        if (v > 0) {
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int i0 = ch * 32 + 2 * e;
            const float2 x = ffma2(make_float2(sv[i0], sv[i0 + 1]), c2, nm2);
            float2 p;
            p.x = ex2_approx(x.x);
            p.y = ex2_approx(x.y);
            if (e & 1) ps1 = fadd2(ps1, p); else ps0 = fadd2(ps0, p);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(p.x, p.y);
            pk[e] = __uint_as_float(*reinterpret_cast<uint32_t*>(&b2));
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0.f;
        }
        tmem_st16(t_row + s_col + ch * 16, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      named_bar_sync(kNbP + wg, kNbPThreads);              // hand P_l to the PV thread
      if (threadIdx.x == 128) LF_TR(10, l);
      l_run += (ps0.x + ps0.y) + (ps1.x + ps1.y);
      m_run = m_new;
      if (threadIdx.x == 128) LF_TR(11, l);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarDone], 0, s_abort, P.wait_limit_ns)) && ok;
    // merge the two groups' partial softmax states: O = sum_w 2^(m_w - m) O_w / l
    s_red[wg * 128 + r] = m_run;
    s_red[256 + wg * 128 + r] = l_run;
    named_bar_sync(kNbEpilogue, kSoftmaxWarps * 32);
    const float m_o = s_red[(wg ^ 1) * 128 + r], l_o = s_red[256 + (wg ^ 1) * 128 + r];
    const float m_all = fmaxf(m_run, m_o);
    const float w_me = m_run == -INFINITY ? 0.f : exp2f(m_run - m_all);
    const float w_o = m_o == -INFINITY ? 0.f : exp2f(m_o - m_all);
    const float l_tot = l_run * w_me + l_o * w_o;
    if (ok) {
      tc_fence_after();
      int qb, i;
      if (BLK == 64) { qb = r < 64 ? qbA : qbB; i = r & 63; }
      else { qb = qbA; i = r; }
      const bool valid = qb >= 0 && i < block_len(D, qb % D.nbpf);
      const int tok = qb >= 0 ? (qb / D.nbpf) * D.T + (qb % D.nbpf) * BLK + i : 0;
      // a whole tile is normalised here; a piece keeps sum_w 2^(m_w - m) O_w, m and l
      const float inv_l = piece < 0 ? 1.0f / l_tot : 1.0f;
      // this group writes output columns [wg*HD/2, (wg+1)*HD/2) from both accumulators
      const float w0 = (wg == 0 ? w_me : w_o) * inv_l, w1 = (wg == 0 ? w_o : w_me) * inv_l;
      const int unit = tail * P.pieces + piece;
      __nv_bfloat16* orow = P.out + ((size_t)tok * D.H + h) * HD + wg * (HD / 2);
      float* prow = P.part_o + ((size_t)unit * 128 + r) * HD + wg * (HD / 2);
#pragma unroll
      for (int ch = 0; ch < HD / 64; ++ch) {
        float a[32], b[32];
        const uint32_t col = wg * (HD / 2) + ch * 32;
        tmem_ld32(t_row + L::kColO0 + col, a);
        tmem_ld32(t_row + L::kColO1 + col, b);
        tmem_ld_wait();
        reg_fence32(a);
        reg_fence32(b);
        float x[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          // a group that never accumulated has weight 0 and its O is not read into the sum
          x[e] = (w0 > 0.f ? a[e] * w0 : 0.f) + (w1 > 0.f ? b[e] * w1 : 0.f);
        if (piece < 0) {
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint32_t pw[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(x[8 * e + 2 * k], x[8 * e + 2 * k + 1]);
                pw[k] = *reinterpret_cast<uint32_t*>(&b2);
              }
              dst[e] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            }
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(prow + ch * 32);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(x[4 * e], x[4 * e + 1], x[4 * e + 2], x[4 * e + 3]);
        }
      }
      if (piece < 0) {
        if (valid && wg == 0 && P.lse != nullptr)
          P.lse[(size_t)h * D.ncur + tok] = (m_all + log2f(l_tot)) * 0.6931471805599453f;
      } else if (wg == 0) {
        P.part_ml[((size_t)unit * 2) * 128 + r] = m_all;
        P.part_ml[((size_t)unit * 2 + 1) * 128 + r] = l_tot;
      }
      tc_fence_before();
    }
  }
  }
  __syncthreads();
  if (threadIdx.x == 0) LF_TR_CTA(2, globaltimer_ns());
  if (warp == 1) {
    // everything the MMA thread issued is complete before tensor memory is released
    if (lane == 0) mbar_wait_drain(&bars[kBarDone], 0, P.wait_limit_ns);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Combines the partial softmax states of the pieces of each tail tile (fixed order):
// m = max_k m_k, l = sum_k 2^(m_k - m) l_k, O = sum_k 2^(m_k - m) O_k / l.
// CTA = (tail tile, group of kMergeRows rows); one thread per (row, 4 channels).
constexpr int kMergeRows = 8;
constexpr int kMaxPieces = 16;     // key ranges a tail tile is split into, at most

__global__ void __launch_bounds__(256)
merge_kernel(const AttnParams P, const Dims D, int HD) {
  const int tail = blockIdx.x;
  const int tile = P.n_whole + tail;
  const int h = tile / P.tiles_per_head, t = tile % P.tiles_per_head;
  const int qbA = D.B == 64 ? 2 * t : t;
  const int qbB = (D.B == 64 && 2 * t + 1 < D.nqb) ? 2 * t + 1 : -1;
  const int c4n = HD / 4;
  for (int idx = threadIdx.x; idx < kMergeRows * c4n; idx += blockDim.x) {
    const int r = blockIdx.y * kMergeRows + idx / c4n, c4 = idx % c4n;
    int qb, i;
    if (D.B == 64) { qb = r < 64 ? qbA : qbB; i = r & 63; }
    else { qb = qbA; i = r; }
    if (qb < 0 || i >= block_len(D, qb % D.nbpf)) continue;
    const int tok = (qb / D.nbpf) * D.T + (qb % D.nbpf) * D.B + i;
    // every piece's state loaded at once (the loads are independent), then combined in
    // piece order
    float mk[kMaxPieces], lk[kMaxPieces];
    float4 xk[kMaxPieces];
#pragma unroll
    for (int k = 0; k < kMaxPieces; ++k) {
      mk[k] = -INFINITY;
      lk[k] = 0.f;
      xk[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k < P.pieces) {
        const size_t unit = (size_t)tail * P.pieces + k;
        mk[k] = P.part_ml[(unit * 2) * 128 + r];
        lk[k] = P.part_ml[(unit * 2 + 1) * 128 + r];
        xk[k] = reinterpret_cast<const float4*>(P.part_o + (unit * 128 + r) * HD)[c4];
      }
    }
    float m = -INFINITY;
#pragma unroll
    for (int k = 0; k < kMaxPieces; ++k) m = fmaxf(m, mk[k]);
    float l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kMaxPieces; ++k) {
      if (mk[k] == -INFINITY) continue;          // a piece with no valid key (or past P.pieces)
      const float w = exp2f(mk[k] - m);
      l += w * lk[k];
      o.x += w * xk[k].x; o.y += w * xk[k].y; o.z += w * xk[k].z; o.w += w * xk[k].w;
    }
    const float inv = 1.0f / l;
    __nv_bfloat162 a = __floats2bfloat162_rn(o.x * inv, o.y * inv);
    __nv_bfloat162 b = __floats2bfloat162_rn(o.z * inv, o.w * inv);
    uint2 pk = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
    reinterpret_cast<uint2*>(P.out + ((size_t)tok * D.H + h) * HD)[c4] = pk;
    if (c4 == 0 && P.lse != nullptr)
      P.lse[(size_t)h * D.ncur + tok] = (m + log2f(l)) * 0.6931471805599453f;
  }
}

}  // namespace lf
