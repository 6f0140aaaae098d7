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
//   * warp 0 streams K tiles and warp 2 V tiles with TMA (128-byte swizzle, zero fill out
//     of bounds), two stages each; warp 1 issues tcgen05.mma: S = Q K^T into one of two
//     tensor-memory buffers, O += P V into a tensor-memory accumulator;
//   * warps 4-7 run the fp32 online softmax, one query row per thread (the row's tensor
//     memory lane): S from tensor memory, P as bf16 into shared memory, O rescaled in
//     tensor memory only when the row maximum grows by more than 2^8 (lazy rescale);
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
// bits 16-27 = frame position (sinks first, then history frames).
__host__ __device__ inline uint32_t plan_pack(int p, int b, uint32_t mask) {
  return ((uint32_t)p << 16) | ((uint32_t)b << 4) | mask;
}

__host__ __device__ inline int tile_count(const Dims& D) {
  return D.B == 64 ? cdiv(D.nqb, 2) : D.nqb;
}
__host__ __device__ inline int plan_stride(const Dims& D) {
  return D.S * D.nbpf + (D.B == 64 ? 2 : 1) * D.nsel;
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

__global__ void __launch_bounds__(32)
plan_kernel(const int32_t* __restrict__ block_idx, uint32_t* __restrict__ plan,
            int32_t* __restrict__ plan_cnt, const Dims D) {
  __shared__ int32_t sa[LF_MAX_SELECTED], sb[LF_MAX_SELECTED];
  const int t = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  const int ntiles = tile_count(D);
  uint32_t* out = plan + ((size_t)h * ntiles + t) * plan_stride(D);
  const int nsink = D.S * D.nbpf;
  for (int e = lane; e < nsink; e += 32) out[e] = plan_pack(e / D.nbpf, e % D.nbpf, 3u);
  int cnt = nsink;
  if (D.F > 0 && D.nsel > 0 && block_idx != nullptr) {
    const int qa = D.B == 64 ? 2 * t : t;
    const int qbB = (D.B == 64 && 2 * t + 1 < D.nqb) ? 2 * t + 1 : -1;
    const int nA = D.nsel, nB = qbB >= 0 ? D.nsel : 0;
    const int32_t* A = block_idx + ((size_t)h * D.nqb + qa) * D.nsel;
    const int32_t* B = qbB >= 0 ? block_idx + ((size_t)h * D.nqb + qbB) * D.nsel : nullptr;
    const int lim = D.F * D.nbpf;
    bool bad = false;
    for (int i = lane; i < nA; i += 32) sa[i] = A[i];
    for (int i = lane; i < nB; i += 32) sb[i] = B[i];
    __syncwarp();
    for (int i = lane; i < nA; i += 32)
      bad |= sa[i] < 0 || sa[i] >= lim || (i > 0 && sa[i - 1] >= sa[i]);
    for (int i = lane; i < nB; i += 32)
      bad |= sb[i] < 0 || sb[i] >= lim || (i > 0 && sb[i - 1] >= sb[i]);
    if (__any_sync(0xffffffffu, bad)) {
      if (lane == 0) record_status(LF_ERR_BAD_INDEX);
    } else {
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
          out[nsink + pos] = plan_pack(D.S + a / D.nbpf, a % D.nbpf, inB ? 3u : 1u);
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
          out[nsink + pos] = plan_pack(D.S + b / D.nbpf, b % D.nbpf, 2u);
        }
        carry += __popc(bal);
      }
      cnt = nsink + nA + nB - ncommon;
    }
  }
  if (lane == 0) plan_cnt[(size_t)h * ntiles + t] = cnt;
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
  int slots[LF_MAX_FRAMES];   // cache slot of frame position p (sinks, then history)
};

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
  static constexpr int kNumBars = 2 * kSlots + 8;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;       // slack for 1024-byte alignment
  // tensor-memory columns: two O accumulators (one per softmax warpgroup), two S buffers;
  // P (bf16 pairs) overwrites the first 64 columns of the S buffer it was computed from
  static constexpr uint32_t kColO0 = 0, kColO1 = 128, kColS0 = 256, kColS1 = 384,
                            kTmemCols = 512;
};

// barrier indices: ring full/empty barriers follow these
enum BarId { kBarQ = 0, kBarSFull = 1, kBarPFull = 3, kBarDone = 5, kBarRing = 6 };

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

constexpr int kSoftmaxWarps = 8;          // two warpgroups, alternate key tiles
// Register split: launched at 168 per thread (384 threads); the load/MMA warpgroup gives
// registers to the two softmax warpgroups: 128 x 72 + 256 x 216 <= 384 x 168.
constexpr int kLaunchRegs = 168, kLowRegs = 72, kHighRegs = 216;
static_assert(128 * kLowRegs + 256 * kHighRegs <= kAttnThreads * kLaunchRegs, "register split");

template <int HD, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const __grid_constant__ AttnParams P, const Dims D) {
  using L = AttnLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* s_plan = reinterpret_cast<uint32_t*>(smem + L::kPlan);
  float* s_red = reinterpret_cast<float*>(smem + L::kRed);
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x, h = blockIdx.y;
  const int ntiles = gridDim.x;

  // query blocks of this tile
  const int qbA = BLK == 64 ? 2 * t : t;
  const int qbB = (BLK == 64 && 2 * t + 1 < D.nqb) ? 2 * t + 1 : -1;
  const int tokA = (qbA / D.nbpf) * D.T + (qbA % D.nbpf) * BLK;
  const int tokB = qbB >= 0 ? (qbB / D.nbpf) * D.T + (qbB % D.nbpf) * BLK : D.ncur;

  const int cnt = P.plan_cnt[(size_t)h * ntiles + t];
  const int n_dense = cdiv(D.ncur, 128);
  const int n_sparse = BLK == 64 ? cdiv(cnt, 2) : cnt;
  const int n_iter = n_dense + n_sparse;

  if (threadIdx.x == 0) {
    mbar_init(&bars[kBarQ], 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kBarSFull + s], 1);
      mbar_init(&bars[kBarPFull + s], 4);
    }
    for (int q = 0; q < 2 * L::kSlots; ++q) mbar_init(&bars[kBarRing + q], 1);
    mbar_init(&bars[kBarDone], 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 3) {
    const uint32_t* src = P.plan + ((size_t)h * ntiles + t) * plan_stride(D);
    for (int i = lane; i < cnt; i += 32) s_plan[i] = src[i];
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&P.tm_q); prefetch_tmap(&P.tm_kc); prefetch_tmap(&P.tm_kh);
    prefetch_tmap(&P.tm_vc); prefetch_tmap(&P.tm_vh);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp < 4) {
  regs_dec<kLowRegs>();
  // -------------------------------------------------------------- producer
  if (warp == 0 && lane == 0) {
    uint64_t* full = &bars[kBarRing];
    uint64_t* empty = &bars[kBarRing + L::kSlots];
    mbar_arrive_expect_tx(&bars[kBarQ], L::kQBytes);
    for (int c = 0; c < L::NH; ++c) {
      uint8_t* dst = smem + L::kQ + c * L::kRegion;
      tma_load_2d(dst, &P.tm_q, &bars[kBarQ], h * HD + c * 64, tokA);
      tma_load_2d(dst + 64 * 128, &P.tm_q, &bars[kBarQ], h * HD + c * 64,
                  BLK == 64 ? tokB : tokA + 64);
    }
    const int n_pos = 2 * n_iter + 1;               // V_{n-1} sits at position 2n
    int q = 0;
    for (; q < n_pos; ++q) {
      bool isK;
      const int j = ring_tile(q, isK);
      const int slot = q % L::kSlots;
      const int rnd = q / L::kSlots;
      if (isK && j >= n_iter) continue;            // no slot used, nothing to load
      if (rnd > 0 && !mbar_wait(&empty[slot], (rnd & 1) ^ 1, s_abort)) break;
      LF_TR(isK ? 0 : 1, j);
      mbar_arrive_expect_tx(&full[slot], L::kStageBytes);
      uint8_t* st = smem + L::kRing + slot * L::kStageBytes;
      const CUtensorMap* tm_cur = isK ? &P.tm_kc : &P.tm_vc;
      const CUtensorMap* tm_hist = isK ? &P.tm_kh : &P.tm_vh;
      for (int box = 0; box < 2; ++box) {
        if (j < n_dense) {
          const int row = j * 128 + box * 64;
          for (int c = 0; c < L::NH; ++c)
            tma_load_2d(st + c * L::kRegion + box * 64 * 128, tm_cur, &full[slot],
                        h * HD + c * 64, row);
        } else {
          const int u = j - n_dense;
          int slot_id = 0, tok = D.T;                   // default: all rows out of bounds
          const int e = BLK == 64 ? 2 * u + box : u;
          if (e < cnt) {
            const uint32_t pe = s_plan[e];
            slot_id = P.slots[pe >> 16];
            tok = (int)((pe >> 4) & 0xFFFu) * BLK + (BLK == 64 ? 0 : box * 64);
          }
          for (int c = 0; c < L::NH; ++c)
            tma_load_3d(st + c * L::kRegion + box * 64 * 128, tm_hist, &full[slot],
                        h * HD + c * 64, tok, slot_id);
        }
      }
    }
    // drain: every load issued must land before the CTA may exit (the last kSlots
    // positions hold the only loads that nobody may have waited for)
    for (int x = max(0, q - L::kSlots); x < q; ++x) {
      bool isK;
      const int jx = ring_tile(x, isK);
      if (!(isK && jx >= n_iter)) mbar_wait_drain(&full[x % L::kSlots], (x / L::kSlots) & 1);
    }
  }
  // -------------------------------------------------------------- MMA issuer
  // Order: S0, S1, then for each i: PV_i (O_{i&1} += P_i V_i), S_{i+2} into the S buffer
  // P_i was read from.  tcgen05.mma runs in issue order, so S_{i+2} overwrites P_i only
  // after PV_i has consumed it, and the completion of S_{i+2} implies that of PV_i.
  else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, HD, 0, 1);
    const uint32_t q_base = smem_u32(smem + L::kQ);
    const uint32_t ring_base = smem_u32(smem + L::kRing);
    uint64_t* full = &bars[kBarRing];
    uint64_t* empty = &bars[kBarRing + L::kSlots];
    auto issue_s = [&](int j) -> bool {
      const int s = j & 1;
      const int q = ring_pos_k(j), slot = q % L::kSlots;
      LF_TR(2, j);
      if (!mbar_wait(&full[slot], (q / L::kSlots) & 1, s_abort)) return false;
      LF_TR(3, j);
      tc_fence_after();
      const uint32_t d_tmem = tmem + (s ? L::kColS1 : L::kColS0);
      const uint32_t k_addr = ring_base + slot * L::kStageBytes;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        const uint32_t off = (ks >> 2) * L::kRegion + (ks & 3) * 32;
        mma_bf16_ss(d_tmem, smem_desc_sw128(q_base + off, 16, 1024),
                    smem_desc_sw128(k_addr + off, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
      }
      mma_commit(&bars[kBarSFull + s]);
      mma_commit(&empty[slot]);
      return true;
    };
    bool ok = mbar_wait(&bars[kBarQ], 0, s_abort);
    if (ok) ok = issue_s(0);
    if (ok && n_iter > 1) ok = issue_s(1);
    for (int i = 0; ok && i < n_iter; ++i) {
      const int s = i & 1;
      const int qv = ring_pos_v(i), vslot = qv % L::kSlots;
      ok = mbar_wait(&full[vslot], (qv / L::kSlots) & 1, s_abort);
      LF_TR(4, i);
      if (ok) ok = mbar_wait(&bars[kBarPFull + s], (i >> 1) & 1, s_abort);
      if (!ok) break;
      LF_TR(5, i);
      tc_fence_after();
      const uint32_t p_tmem = tmem + (s ? L::kColS1 : L::kColS0);
      const uint32_t o_tmem = tmem + (s ? L::kColO1 : L::kColO0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)            // 128 keys, 16 per MMA, 8 columns each
        mma_bf16_ts(o_tmem, p_tmem + ks * 8,
                    smem_desc_sw128(ring_base + vslot * L::kStageBytes + ks * 16 * 128,
                                    L::kRegion, 1024),
                    idesc_pv, (i >= 2 || ks > 0) ? 1u : 0u);
      mma_commit(&empty[vslot]);
      if (i + 2 < n_iter) ok = issue_s(i + 2);
    }
    // completion of everything issued: epilogue may read O, tensor memory may be freed
    mma_commit(&bars[kBarDone]);
  }
  } else {
  regs_inc<kHighRegs>();
  // -------------------------------------------------------------- softmax + epilogue
  {
    const int wg = (warp - 4) >> 2;                        // handles key tiles j = wg, wg+2, ...
    const int r = (threadIdx.x - 128) & 127;               // query row = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t row_bit = (BLK == 64 && r >= 64) ? 2u : 1u;
    const uint32_t s_col = wg ? L::kColS1 : L::kColS0;
    const uint32_t o_col = wg ? L::kColO1 : L::kColO0;
    const float c = D.scale * 1.4426950408889634f;         // scale * log2(e)
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int n_mine = 0;                                        // PVs into this group's O
    for (int j = wg; j < n_iter; j += 2, ++n_mine) {
      if (threadIdx.x == 128) LF_TR(6, j);
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull + wg], (j >> 1) & 1, s_abort)) && ok;
      if (threadIdx.x == 128) LF_TR(7, j);
      tc_fence_after();
      float sv[128];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32(t_row + s_col + ch * 32, sv + ch * 32);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) reg_fence32(sv + ch * 32);
      if (threadIdx.x == 128) LF_TR(8, j);

      // valid key columns of this row: [0, v0) and [64, 64 + v1)
      int v0, v1;
      if (j < n_dense) {
        const int n = min(128, D.ncur - j * 128);
        v0 = min(64, n);
        v1 = max(0, n - 64);
      } else {
        const int u = j - n_dense;
        if (BLK == 64) {
          v0 = v1 = 0;
          if (2 * u < cnt) {
            const uint32_t e = s_plan[2 * u];
            if (e & row_bit) v0 = block_len(D, (e >> 4) & 0xFFF);
          }
          if (2 * u + 1 < cnt) {
            const uint32_t e = s_plan[2 * u + 1];
            if (e & row_bit) v1 = block_len(D, (e >> 4) & 0xFFF);
          }
        } else {
          const uint32_t e = s_plan[u];
          const int len = (e & row_bit) ? block_len(D, (e >> 4) & 0xFFF) : 0;
          v0 = min(64, len);
          v1 = max(0, len - 64);
        }
      }
      if (v0 < 64 || v1 < 64) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          if (i >= v0) sv[i] = -INFINITY;
          if (i >= v1) sv[64 + i] = -INFINITY;
        }
      }
      float mx8[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmax3f(sv[k], sv[8 + k], sv[16 + k]);
#pragma unroll
      for (int i = 24; i < 120; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmax3f(mx8[k], sv[i + k], sv[i + 8 + k]);
#pragma unroll
      for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(mx8[k], sv[120 + k]);
      const float m_tile = fmaxf(fmax3f(mx8[0], mx8[1], mx8[2]),
                                 fmax3f(fmax3f(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7])) * c;
      float m_new = m_run;
      bool resc = false;
      if (m_tile > m_run + 8.0f) { m_new = m_tile; resc = true; }
      // lazy rescale of this group's O: its previous PV (PV_{j-2}) completed before S_j did
      if (n_mine > 0 && __any_sync(0xffffffffu, resc)) {
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
      if (threadIdx.x == 128) LF_TR(9, j);
      const float mref = (m_new == -INFINITY) ? 0.f : m_new;
      float ps[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = ex2_approx(fmaf(sv[half * 64 + 2 * e], c, -mref));
          const float p1 = ex2_approx(fmaf(sv[half * 64 + 2 * e + 1], c, -mref));
          ps[e & 3] += p0 + p1;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[e] = __uint_as_float(*reinterpret_cast<uint32_t*>(&b2));
        }
        tmem_st32(t_row + s_col + half * 32, pk);
      }
      if (threadIdx.x == 128) LF_TR(10, j);
      tmem_st_wait();
      l_run += (ps[0] + ps[1]) + (ps[2] + ps[3]);
      m_run = m_new;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarPFull + wg]);
      if (threadIdx.x == 128) LF_TR(11, j);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarDone], 0, s_abort)) && ok;
    // merge the two groups' partial softmax states: O = sum_w 2^(m_w - m) O_w / l
    s_red[wg * 128 + r] = m_run;
    s_red[256 + wg * 128 + r] = l_run;
    named_bar_sync(1, kSoftmaxWarps * 32);
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
      const float inv_l = 1.0f / l_tot;
      // this group writes output columns [wg*HD/2, (wg+1)*HD/2) from both accumulators
      const float w0 = (wg == 0 ? w_me : w_o) * inv_l, w1 = (wg == 0 ? w_o : w_me) * inv_l;
      __nv_bfloat16* orow = P.out + ((size_t)tok * D.H + h) * HD + wg * (HD / 2);
#pragma unroll
      for (int ch = 0; ch < HD / 64; ++ch) {
        float a[32], b[32];
        const uint32_t col = wg * (HD / 2) + ch * 32;
        tmem_ld32(t_row + L::kColO0 + col, a);
        tmem_ld32(t_row + L::kColO1 + col, b);
        tmem_ld_wait();
        reg_fence32(a);
        reg_fence32(b);
        if (valid) {
          uint32_t pw[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            // a group that never accumulated has weight 0 and its O is not read into the sum
            const float x0 = (w0 > 0.f ? a[2 * e] * w0 : 0.f) + (w1 > 0.f ? b[2 * e] * w1 : 0.f);
            const float x1 = (w0 > 0.f ? a[2 * e + 1] * w0 : 0.f) +
                             (w1 > 0.f ? b[2 * e + 1] * w1 : 0.f);
            __nv_bfloat162 b2 = __floats2bfloat162_rn(x0, x1);
            pw[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pw[4 * e], pw[4 * e + 1], pw[4 * e + 2], pw[4 * e + 3]);
        }
      }
      if (valid && wg == 0 && P.lse != nullptr)
        P.lse[(size_t)h * D.ncur + tok] = (m_all + log2f(l_tot)) * 0.6931471805599453f;
      tc_fence_before();
    }
  }
  }
  __syncthreads();
  if (warp == 1) {
    // everything the MMA thread issued is complete before tensor memory is released
    if (lane == 0) mbar_wait_drain(&bars[kBarDone], 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace lf
