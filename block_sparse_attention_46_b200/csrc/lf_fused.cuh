// lf_fused.cuh — stages (b) and (c) for the one-call paths (lf_select_chunk,
// lf_forward_chunk): every history block's score against every pooled query block (a
// small GEMM, q_blk . k_blk^T, fixed summation order), then per group of query blocks the
// frame scores from them by linearity (a frame's pooled key is the length-weighted mean of
// its block keys, so its score is the length-weighted mean of the block scores), the
// top-k_f frames, the top-k_b blocks in each chosen frame, and the key plans of the
// group's query tiles.  [LF-gist 2.2] two-stage mask selection; [LF-yly 三] inner-product
// similarity.
#pragma once
#include "lf_select.cuh"
#include "lf_attn.cuh"

namespace lf {

#ifndef LF_FUSE_QB
#define LF_FUSE_QB 2
#endif
#ifndef LF_SCORE_QB
#define LF_SCORE_QB 16
#endif
constexpr int kFuseQb = LF_FUSE_QB;        // query blocks per CTA (even: whole tile pairs)
constexpr int kFuseMaxBlocks = 2048;       // F * n_bpf handled by the fused path
constexpr int kFuseMaxSel = 256;           // k_f * k_b handled by the fused path

__host__ __device__ inline bool fused_select_ok(const Dims& D) {
  return D.F > 0 && D.F * D.nbpf <= kFuseMaxBlocks && D.nsel <= kFuseMaxSel &&
         D.F <= 32 * kMaxPerLane && D.nbpf <= 32 * kMaxPerLane;
}

__host__ __device__ inline size_t fused_select_smem(const Dims& D) {
  return (size_t)kFuseQb * D.F * D.nbpf * 4 + (size_t)kFuseQb * D.nsel * 4 +
         (size_t)kFuseQb * D.kf * 4;
}

// Scores of every history block against every pooled query block of head h:
// s[h, qb, r] = q_blk[h, qb] . k_blk[h, r], r = f * n_bpf + b.  CTA = (64 rows, head,
// kScoreQb query blocks); rows and queries are staged in shared memory with coalesced
// loads; thread (row, quarter) computes kScoreQb / 4 query blocks against one row, each
// score one fixed-order sum over the channels.
constexpr int kScoreRows = 64, kScoreQb = LF_SCORE_QB;
constexpr int kScoreQpt = kScoreQb * kScoreRows / 256;    // query blocks per thread
static_assert(kScoreQpt >= 1 && kScoreQpt * 256 == kScoreQb * kScoreRows, "score tiling");

struct ScoreArgs {
  const float* q_blk;   // [H, nqb, d]
  const float* k_blk;   // [H, F, nbpf, d], or null when k_pool is used
  const float* k_pool;  // [n_slots, H, nbpf, d] pooled-key cache, read through slots[]
  float* scores;        // [H, nqb, F * nbpf]
  int slots[LF_MAX_FRAMES];
};

template <int HD>
__global__ void __launch_bounds__(256)   // staging assumes exactly 256 threads
block_scores_kernel(const __grid_constant__ ScoreArgs a, const Dims D) {
  const float* __restrict__ q_blk = a.q_blk;
  float* __restrict__ scores = a.scores;
  __shared__ float4 sk4[kScoreRows * (HD / 4 + 1)];
  __shared__ float4 sq4[kScoreQb * (HD / 4)];
  const int NB = D.F * D.nbpf;
  const int r0 = blockIdx.x * kScoreRows, h = blockIdx.y, q0 = blockIdx.z * kScoreQb;
  const int pitch = HD / 4 + 1;                       // float4 pitch, padded
  {
    // kScoreRows * HD / 4 float4 = 2048 (d = 128): eight loads in flight per thread
    constexpr int n4 = kScoreRows * (HD / 4);
    float4 v[n4 / 256];
#pragma unroll
    for (int u = 0; u < n4 / 256; ++u) {
      const int i = threadIdx.x + u * 256, r = i / (HD / 4), c4 = i % (HD / 4);
      const int rr = r0 + r;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (rr < NB) {
        const float* row = a.k_pool != nullptr
            ? a.k_pool + (((size_t)a.slots[rr / D.nbpf] * D.H + h) * D.nbpf + rr % D.nbpf) * HD
            : a.k_blk + ((size_t)h * NB + rr) * HD;
        v[u] = __ldg(reinterpret_cast<const float4*>(row) + c4);
      }
    }
#pragma unroll
    for (int u = 0; u < n4 / 256; ++u) {
      const int i = threadIdx.x + u * 256, r = i / (HD / 4), c4 = i % (HD / 4);
      sk4[r * pitch + c4] = v[u];
    }
  }
  for (int i = threadIdx.x; i < kScoreQb * (HD / 4); i += 256) {
    const int g = i / (HD / 4), c4 = i % (HD / 4);
    sq4[i] = q0 + g < D.nqb
        ? __ldg(reinterpret_cast<const float4*>(q_blk + ((size_t)h * D.nqb + q0 + g) * HD) + c4)
        : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  const int r = threadIdx.x % kScoreRows, gq = threadIdx.x / kScoreRows;   // 4 quarters
  float acc[kScoreQpt];
#pragma unroll
  for (int u = 0; u < kScoreQpt; ++u) acc[u] = 0.f;
#pragma unroll 8
  for (int c4 = 0; c4 < HD / 4; ++c4) {
    const float4 k = sk4[r * pitch + c4];
#pragma unroll
    for (int u = 0; u < kScoreQpt; ++u) {
      const float4 q = sq4[(gq * kScoreQpt + u) * (HD / 4) + c4];
      acc[u] = fmaf(q.x, k.x, acc[u]); acc[u] = fmaf(q.y, k.y, acc[u]);
      acc[u] = fmaf(q.z, k.z, acc[u]); acc[u] = fmaf(q.w, k.w, acc[u]);
    }
  }
  if (r0 + r < NB)
#pragma unroll
    for (int u = 0; u < kScoreQpt; ++u) {
      const int qb = q0 + gq * kScoreQpt + u;
      if (qb < D.nqb) scores[((size_t)h * D.nqb + qb) * NB + r0 + r] = acc[u];
    }
}

// Per (head, group of kFuseQb query blocks): frame scores by linearity from the block
// scores, frame top-k, block top-k in each chosen frame, block_idx, and the key plans of
// the group's query tiles.
__global__ void __launch_bounds__(256)
select_pick_kernel(const float* __restrict__ scores, int32_t* __restrict__ block_idx,
                   uint32_t* __restrict__ plan, int32_t* __restrict__ plan_cnt, const Dims D) {
  extern __shared__ float4 sm4[];
  const int NB = D.F * D.nbpf;
  float* sc = reinterpret_cast<float*>(sm4);                        // [kFuseQb][NB]
  int32_t* sl = reinterpret_cast<int32_t*>(sc + (size_t)kFuseQb * NB);   // [kFuseQb][nsel]
  int32_t* sf = sl + kFuseQb * D.nsel;                              // [kFuseQb][kf]
  const int h = blockIdx.y, qb0 = blockIdx.x * kFuseQb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    // the group's rows of the score matrix are contiguous: [qb0, qb0 + kFuseQb) x NB
    const int ng = min(kFuseQb, D.nqb - qb0);
    stage_words(sc, scores + ((size_t)h * D.nqb + qb0) * NB, ng * NB, threadIdx.x, blockDim.x);
  }
  __syncthreads();

  const float invT = 1.0f / (float)D.T;
  const int nwarps = blockDim.x / 32;
  // frame scores (by linearity from the block scores) and frame top-k: a warp per query block
  for (int g = warp; g < kFuseQb; g += nwarps) {
    if (qb0 + g >= D.nqb) continue;
    const float* s = sc + (size_t)g * NB;
    float fs[kMaxPerLane];
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
      const int f = lane + 32 * j;
      float v = -INFINITY;
      if (f < D.F) {
        v = 0.f;
        for (int b = 0; b < D.nbpf; ++b) v += (float)block_len(D, b) * s[f * D.nbpf + b];
        v *= invT;
      }
      fs[j] = v;
    }
    const uint32_t taken = warp_topk(fs, D.F, D.kf);
    warp_write_ascending(taken, D.F, sf + g * D.kf, 0);
  }
  __syncthreads();
  // block top-k inside each chosen frame: a warp per (query block, chosen frame)
  for (int task = warp; task < kFuseQb * D.kf; task += nwarps) {
    const int g = task / D.kf, j = task % D.kf;
    if (qb0 + g >= D.nqb) continue;
    const float* s = sc + (size_t)g * NB;
    const int f = sf[g * D.kf + j];
    float bs[kMaxPerLane];
#pragma unroll
    for (int u = 0; u < kMaxPerLane; ++u) {
      const int b = lane + 32 * u;
      bs[u] = b < D.nbpf ? s[f * D.nbpf + b] : -INFINITY;
    }
    const uint32_t tb = warp_topk(bs, D.nbpf, D.kb);
    warp_write_ascending(tb, D.nbpf, sl + g * D.nsel + j * D.kb, f * D.nbpf);
  }
  __syncthreads();
  // the lists (chosen frames ascending, blocks ascending inside each): all threads
  for (int i = threadIdx.x; i < kFuseQb * D.nsel; i += blockDim.x) {
    const int g = i / D.nsel, qb = qb0 + g;
    if (qb < D.nqb) block_idx[((size_t)h * D.nqb + qb) * D.nsel + i % D.nsel] = sl[i];
  }

  // key plans of the group's tiles (one warp per tile)
  const int ntiles = tile_count(D);
  const int per = D.B == 64 ? 2 : 1;                       // query blocks per tile
  for (int p = warp; p < kFuseQb / per; p += blockDim.x / 32) {
    const int qa = qb0 + p * per;
    if (qa >= D.nqb) continue;
    const int t = qa / per;
    const bool two = per == 2 && qa + 1 < D.nqb;
    const int cnt = warp_write_plan(sl + (qa - qb0) * D.nsel, D.nsel,
                                    two ? sl + (qa + 1 - qb0) * D.nsel : sl, two ? D.nsel : 0,
                                    plan + ((size_t)h * ntiles + t) * plan_stride(D), D);
    if (lane == 0) plan_cnt[(size_t)h * ntiles + t] = cnt;
  }
}

// One-dimensional selection (no frame stage), the ablation the pages compare against
// [LF-yly 四]: per (head, query block) the K = kf * kb best-scoring history blocks over all
// frames, equal scores to the lower id, written in ascending id order.  One CTA per
// (query block, head): a bitonic sort of the F * n_bpf scores (padded with -inf to n2, a
// power of two) by (score descending, id ascending), then the first K ids are compacted
// in id order by one warp.
constexpr int kTopkThreads = 256;

__global__ void __launch_bounds__(kTopkThreads)
select_topk_kernel(const float* __restrict__ scores, int32_t* __restrict__ block_idx,
                   const Dims D, int n2) {
  extern __shared__ float4 smt4[];
  float* sv = reinterpret_cast<float*>(smt4);     // [n2] scores
  int* si = reinterpret_cast<int*>(sv + n2);      // [n2] ids
  int* mark = si + n2;                            // [n2] 1 = selected
  const int qb = blockIdx.x, h = blockIdx.y;
  const int nb = D.F * D.nbpf, K = D.nsel;
  const float* src = scores + ((size_t)h * D.nqb + qb) * nb;
  for (int i = threadIdx.x; i < n2; i += blockDim.x) {
    sv[i] = i < nb ? src[i] : -INFINITY;
    si[i] = i;
    mark[i] = 0;
  }
  __syncthreads();
  for (int size = 2; size <= n2; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int t = threadIdx.x; t < n2 / 2; t += blockDim.x) {
        const int lo = 2 * t - (t & (stride - 1)), hi = lo + stride;
        const float a = sv[lo], b = sv[hi];
        const int ia = si[lo], ib = si[hi];
        const bool a_first = a > b || (a == b && ia < ib);
        if (a_first != ((lo & size) == 0)) {     // this bitonic run is built the other way
          sv[lo] = b; sv[hi] = a;
          si[lo] = ib; si[hi] = ia;
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < K; i += blockDim.x) mark[si[i]] = 1;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int32_t* dst = block_idx + ((size_t)h * D.nqb + qb) * K;
    int count = 0;
    for (int base = 0; base < nb; base += 32) {
      const bool sel = base + lane < nb && mark[base + lane];
      const uint32_t bal = __ballot_sync(0xffffffffu, sel);
      if (sel) dst[count + __popc(bal & ((1u << lane) - 1u))] = base + lane;
      count += __popc(bal);
    }
  }
}

}  // namespace lf
