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
constexpr int kAttnThreads = 256;

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
  static constexpr int kK = kQ + kQBytes;            // K stages
  static constexpr int kStageBytes = NH * kRegion;
  static constexpr int kV = kK + 2 * kStageBytes;    // V stages
  static constexpr int kP = kV + 2 * kStageBytes;    // P: 2 key halves x 128 rows x 128 B
  static constexpr int kPBytes = 2 * kRegion;
  static constexpr int kPlan = kP + kPBytes;
  static constexpr int kBar = kPlan + kMaxPlan * 4;
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;       // slack for 1024-byte alignment
  // tensor-memory columns
  static constexpr uint32_t kColO = 0, kColS0 = 128, kColS1 = 256, kTmemCols = 512;
};

enum BarId {
  kBarQ = 0, kBarKFull = 1, kBarKEmpty = 3, kBarVFull = 5, kBarVEmpty = 7,
  kBarSFull = 9, kBarSEmpty = 11, kBarPFull = 13, kBarODone = 14, kBarDrain = 15
};

template <int HD, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const __grid_constant__ AttnParams P, const Dims D) {
  using L = AttnLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* s_plan = reinterpret_cast<uint32_t*>(smem + L::kPlan);
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
      mbar_init(&bars[kBarKFull + s], 1);
      mbar_init(&bars[kBarKEmpty + s], 1);
      mbar_init(&bars[kBarVFull + s], 1);
      mbar_init(&bars[kBarVEmpty + s], 1);
      mbar_init(&bars[kBarSFull + s], 1);
      mbar_init(&bars[kBarSEmpty + s], 4);
    }
    mbar_init(&bars[kBarPFull], 4);
    mbar_init(&bars[kBarODone], 1);
    mbar_init(&bars[kBarDrain], 1);
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
  }
  if (warp == 2 && lane == 0) {
    prefetch_tmap(&P.tm_vc); prefetch_tmap(&P.tm_vh);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // -------------------------------------------------------------- producers
  if ((warp == 0 || warp == 2) && lane == 0) {
    const bool isK = warp == 0;
    const CUtensorMap* tm_cur = isK ? &P.tm_kc : &P.tm_vc;
    const CUtensorMap* tm_hist = isK ? &P.tm_kh : &P.tm_vh;
    uint64_t* full = &bars[isK ? kBarKFull : kBarVFull];
    uint64_t* empty = &bars[isK ? kBarKEmpty : kBarVEmpty];
    uint8_t* stage0 = smem + (isK ? L::kK : L::kV);
    if (isK) {
      mbar_arrive_expect_tx(&bars[kBarQ], L::kQBytes);
      for (int c = 0; c < L::NH; ++c) {
        uint8_t* dst = smem + L::kQ + c * L::kRegion;
        tma_load_2d(dst, &P.tm_q, &bars[kBarQ], h * HD + c * 64, tokA);
        tma_load_2d(dst + 64 * 128, &P.tm_q, &bars[kBarQ], h * HD + c * 64,
                    BLK == 64 ? tokB : tokA + 64);
      }
    }
    int j = 0;
    for (; j < n_iter; ++j) {
      const int s = j & 1;
      if (j >= 2 && !mbar_wait(&empty[s], ((j >> 1) & 1) ^ 1, s_abort)) break;
      mbar_arrive_expect_tx(&full[s], L::kStageBytes);
      uint8_t* st = stage0 + s * L::kStageBytes;
      for (int box = 0; box < 2; ++box) {
        if (j < n_dense) {
          const int row = j * 128 + box * 64;
          for (int c = 0; c < L::NH; ++c)
            tma_load_2d(st + c * L::kRegion + box * 64 * 128, tm_cur, &full[s],
                        h * HD + c * 64, row);
        } else {
          const int u = j - n_dense;
          int slot = 0, tok = D.T;                      // default: all rows out of bounds
          const int e = BLK == 64 ? 2 * u + box : u;
          if (e < cnt) {
            const uint32_t pe = s_plan[e];
            slot = P.slots[pe >> 16];
            tok = (int)((pe >> 4) & 0xFFFu) * BLK + (BLK == 64 ? 0 : box * 64);
          }
          for (int c = 0; c < L::NH; ++c)
            tma_load_3d(st + c * L::kRegion + box * 64 * 128, tm_hist, &full[s],
                        h * HD + c * 64, tok, slot);
        }
      }
    }
    // drain: every load issued must land before the CTA may exit
    for (int s = 0; s < 2; ++s) {
      const int last = (j - 1 - s) >= 0 ? ((j - 1 - s) & ~1) + s : -1;
      if (last >= 0) mbar_wait_drain(&full[s], (last >> 1) & 1);
    }
  }
  // -------------------------------------------------------------- MMA issuer
  else if (warp == 1 && lane == 0) {
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, HD, 0, 1);
    const uint32_t q_base = smem_u32(smem + L::kQ);
    const uint32_t k_base = smem_u32(smem + L::kK);
    const uint32_t v_base = smem_u32(smem + L::kV);
    const uint32_t p_base = smem_u32(smem + L::kP);
    bool ok = mbar_wait(&bars[kBarQ], 0, s_abort);
    for (int j = 0; ok && j <= n_iter; ++j) {
      if (j < n_iter) {
        const int s = j & 1;
        ok = mbar_wait(&bars[kBarKFull + s], (j >> 1) & 1, s_abort);
        if (ok && j >= 2) ok = mbar_wait(&bars[kBarSEmpty + s], ((j >> 1) & 1) ^ 1, s_abort);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (s ? L::kColS1 : L::kColS0);
#pragma unroll
        for (int ks = 0; ks < HD / 16; ++ks) {
          const uint32_t off = (ks >> 2) * L::kRegion + (ks & 3) * 32;
          mma_bf16_ss(d_tmem, smem_desc_sw128(q_base + off, 16, 1024),
                      smem_desc_sw128(k_base + s * L::kStageBytes + off, 16, 1024),
                      idesc_qk, ks > 0 ? 1u : 0u);
        }
        mma_commit(&bars[kBarSFull + s]);
        mma_commit(&bars[kBarKEmpty + s]);
      }
      if (j >= 1) {
        const int i = j - 1, s = i & 1;
        ok = mbar_wait(&bars[kBarVFull + s], (i >> 1) & 1, s_abort);
        if (ok) ok = mbar_wait(&bars[kBarPFull], i & 1, s_abort);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {          // 128 keys, 16 per MMA
          const uint32_t a_off = (ks >> 2) * L::kRegion + (ks & 3) * 32;
          const uint32_t b_off = ks * 16 * 128;
          mma_bf16_ss(tmem + L::kColO, smem_desc_sw128(p_base + a_off, 16, 1024),
                      smem_desc_sw128(v_base + s * L::kStageBytes + b_off, L::kRegion, 1024),
                      idesc_pv, (i > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bars[kBarODone]);
        mma_commit(&bars[kBarVEmpty + s]);
      }
    }
    // drain: all MMAs issued by this thread complete before tensor memory is released
    mma_commit(&bars[kBarDrain]);
    mbar_wait_drain(&bars[kBarDrain], 0);
  }
  // -------------------------------------------------------------- softmax + epilogue
  else if (warp >= 4) {
    const int r = threadIdx.x - 128;                       // query row = TMEM lane
    const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t row_bit = (BLK == 64 && r >= 64) ? 2u : 1u;
    const float c = D.scale * 1.4426950408889634f;         // scale * log2(e)
    uint8_t* p_smem = smem + L::kP;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    int j = 0;
    for (; j < n_iter; ++j) {
      const int s = j & 1;
      ok = mbar_wait(&bars[kBarSFull + s], (j >> 1) & 1, s_abort);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      float sv[128];
      const uint32_t s_col = s ? L::kColS1 : L::kColS0;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_ld32(t_row + s_col + ch * 32, sv + ch * 32);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) reg_fence32(sv + ch * 32);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarSEmpty + s]);

      // valid key columns of this row: [0, v0) in the first 64, [64, 64 + v1) in the second
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
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        if (i >= v0) sv[i] = -INFINITY;
        if (i >= v1) sv[64 + i] = -INFINITY;
      }
#pragma unroll
      for (int i = 0; i < 128; ++i) mx = fmaxf(mx, sv[i]);
      const float m_tile = mx * c;
      float m_new = m_run;
      bool resc = false;
      if (m_tile > m_run + 8.0f) { m_new = m_tile; resc = true; }
      const float alpha = (m_new == -INFINITY) ? 1.f : exp2f(m_run - m_new);

      // PV of the previous tile must be done: P buffer reuse and O rescale
      if (j > 0) {
        ok = mbar_wait(&bars[kBarODone], (j - 1) & 1, s_abort);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, resc)) {
          const float a = resc ? alpha : 1.f;
#pragma unroll
          for (int ch = 0; ch < HD / 32; ++ch) {
            float o[32];
            tmem_ld32(t_row + L::kColO + ch * 32, o);
            tmem_ld_wait();
            reg_fence32(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] *= a;
            tmem_st32(t_row + L::kColO + ch * 32, o);
          }
          tmem_st_wait();
        }
      }
      if (resc) l_run *= alpha;
      const float mref = (m_new == -INFINITY) ? 0.f : m_new;
      float psum = 0.f;
      uint8_t* prow = p_smem + r * 128;
#pragma unroll
      for (int kh = 0; kh < 2; ++kh) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float p0 = ex2_approx(fmaf(sv[kh * 64 + cc * 8 + 2 * e], c, -mref));
            const float p1 = ex2_approx(fmaf(sv[kh * 64 + cc * 8 + 2 * e + 1], c, -mref));
            psum += p0 + p1;
            __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
            pk[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          const int chunk = cc ^ (r & 7);
          *reinterpret_cast<uint4*>(prow + kh * L::kRegion + chunk * 16) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      l_run += psum;
      m_run = m_new;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars[kBarPFull]);
    }
    if (ok && n_iter > 0) {
      ok = mbar_wait(&bars[kBarODone], (n_iter - 1) & 1, s_abort);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      // output row
      int qb, i;
      if (BLK == 64) { qb = r < 64 ? qbA : qbB; i = r & 63; }
      else { qb = qbA; i = r; }
      const bool valid = qb >= 0 && i < block_len(D, qb % D.nbpf);
      const int tok = qb >= 0 ? (qb / D.nbpf) * D.T + (qb % D.nbpf) * BLK + i : 0;
      const float inv_l = 1.0f / l_run;
      __nv_bfloat16* orow = P.out + ((size_t)tok * D.H + h) * HD;
#pragma unroll
      for (int ch = 0; ch < HD / 32; ++ch) {
        float o[32];
        tmem_ld32(t_row + L::kColO + ch * 32, o);
        tmem_ld_wait();
        reg_fence32(o);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            __nv_bfloat162 b2 = __floats2bfloat162_rn(o[2 * e] * inv_l, o[2 * e + 1] * inv_l);
            pk[e] = *reinterpret_cast<uint32_t*>(&b2);
          }
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
        }
      }
      if (valid && P.lse != nullptr)
        P.lse[(size_t)h * D.ncur + tok] = (m_run + log2f(l_run)) * 0.6931471805599453f;
      tc_fence_before();
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace lf
