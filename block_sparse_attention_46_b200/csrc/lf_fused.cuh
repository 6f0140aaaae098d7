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
// s[h, qb, r] = q_blk[h, qb] . k_blk[h, r], r = f * n_bpf + b.  CTA = (128 rows, head,
// 16 query blocks), four warps; rows and queries are staged in shared memory with
// coalesced loads and a row pitch of d + 4 floats.  Each thread computes a 4 x 4 tile,
// rows rg + 8i and query blocks qg + 4u (rg = lane % 8, qg = lane / 8): at every step the
// warp reads 8 distinct rows and 4 distinct queries, one 128-byte wavefront each, so the
// loop runs at the FMA rate.  Each score is one fixed-order sum over the channels.
constexpr int kScoreRows = 128, kScoreQb = 16, kScoreThreads = 128;

template <int HD>
__host__ __device__ constexpr size_t score_smem() {
  return (size_t)(kScoreRows + kScoreQb) * (HD / 4 + 1) * sizeof(float4);
}

struct ScoreArgs {
  const float* q_blk;   // [H, nqb, d]
  const float* k_blk;   // [H, F, nbpf, d], or null when k_pool is used
  const float* k_pool;  // [n_slots, H, nbpf, d] pooled-key cache, read through slots[]
  float* scores;        // [H, nqb, F * nbpf]
  int slots[LF_MAX_FRAMES];
};

template <int HD>
__global__ void __launch_bounds__(kScoreThreads)   // staging assumes exactly 128 threads
block_scores_kernel(const __grid_constant__ ScoreArgs a, const Dims D) {
  constexpr int P = HD / 4 + 1;                        // float4 pitch, padded
  extern __shared__ float4 smq4[];
  float4* sk4 = smq4;                                  // [kScoreRows][P]
  float4* sq4 = smq4 + kScoreRows * P;                 // [kScoreQb][P]
  const int NB = D.F * D.nbpf;
  const int r0 = blockIdx.x * kScoreRows, h = blockIdx.y, q0 = blockIdx.z * kScoreQb;
  {
    // kScoreRows * HD / 4 float4 (4096 at d = 128), eight loads in flight per thread
    constexpr int n4 = kScoreRows * (HD / 4), batch = 8;
    static_assert(n4 % (batch * kScoreThreads) == 0, "score staging");
#pragma unroll 1
    for (int i0 = 0; i0 < n4; i0 += batch * kScoreThreads) {
      float4 v[batch];
#pragma unroll
      for (int u = 0; u < batch; ++u) {
        const int i = i0 + threadIdx.x + u * kScoreThreads, r = i / (HD / 4), c4 = i % (HD / 4);
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
      for (int u = 0; u < batch; ++u) {
        const int i = i0 + threadIdx.x + u * kScoreThreads, r = i / (HD / 4), c4 = i % (HD / 4);
        sk4[r * P + c4] = v[u];
      }
    }
  }
  for (int i = threadIdx.x; i < kScoreQb * (HD / 4); i += kScoreThreads) {
    const int g = i / (HD / 4), c4 = i % (HD / 4);
    sq4[g * P + c4] = q0 + g < D.nqb
        ? __ldg(reinterpret_cast<const float4*>(a.q_blk + ((size_t)h * D.nqb + q0 + g) * HD) + c4)
        : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rg = lane & 7, qg = lane >> 3;
  const int rb = warp * 32 + rg;                       // rows rb + 8i, i < 4
  float acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[u][i] = 0.f;
#pragma unroll 4
  for (int c4 = 0; c4 < HD / 4; ++c4) {
    float4 k[4], q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) k[i] = sk4[(rb + 8 * i) * P + c4];
#pragma unroll
    for (int u = 0; u < 4; ++u) q[u] = sq4[(qg + 4 * u) * P + c4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float t = acc[u][i];
        t = fmaf(q[u].x, k[i].x, t); t = fmaf(q[u].y, k[i].y, t);
        t = fmaf(q[u].z, k[i].z, t); t = fmaf(q[u].w, k[i].w, t);
        acc[u][i] = t;
      }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int qb = q0 + qg + 4 * u;
    if (qb >= D.nqb) continue;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = r0 + rb + 8 * i;
      if (r < NB) a.scores[((size_t)h * D.nqb + qb) * NB + r] = acc[u][i];
    }
  }
}

// Per (head, group of kFuseQb query blocks): frame scores by linearity from the block
// scores, frame top-k, block top-k in each chosen frame, block_idx, and the key plans of
// the group's query tiles.  A tile's plan is written by the whole CTA from two bitmaps
// over the F * n_bpf history blocks (one per query block of the tile): the union's bits
// in id order give the entries, a prefix count of the union's words their positions.
constexpr int kPickThreads = 256;
constexpr int kFuseWords = kFuseMaxBlocks / 32;

// The pick of one group of kFuseQb query blocks of head h (qb0 = first), by a whole CTA of
// kPickThreads threads; `sm` is dynamic shared memory of at least fused_select_smem(D)
// bytes.  Score rows are read with L2-coherent loads (they may have been written by other
// CTAs of the same launch).  plan == nullptr: the lists only.
__device__ __forceinline__ void pick_group(const float* __restrict__ scores,
                                           int32_t* __restrict__ block_idx,
                                           uint32_t* __restrict__ plan,
                                           int32_t* __restrict__ plan_cnt, const Dims& D, int h,
                                           int qb0, float* sm) {
  const int NB = D.F * D.nbpf;
  float* sc = sm;                                                   // [kFuseQb][NB]
  int32_t* sl = reinterpret_cast<int32_t*>(sc + (size_t)kFuseQb * NB);   // [kFuseQb][nsel]
  int32_t* sf = sl + kFuseQb * D.nsel;                              // [kFuseQb][kf]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    // the group's rows of the score matrix are contiguous: [qb0, qb0 + kFuseQb) x NB
    const int ng = min(kFuseQb, D.nqb - qb0);
    const float* src = scores + ((size_t)h * D.nqb + qb0) * NB;
    const int n = ng * NB, tid = threadIdx.x, nt = blockDim.x;
    int i = tid;
    for (; i + 7 * nt < n; i += 8 * nt) {          // eight L2 loads in flight per thread
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(src + i + u * nt);
#pragma unroll
      for (int u = 0; u < 8; ++u) sc[i + u * nt] = v[u];
    }
    for (; i < n; i += nt) sc[i] = __ldcg(src + i);
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
  if (plan == nullptr) return;                             // lists only

  // key plans of the group's tiles
  __shared__ uint32_t s_bits[2][kFuseWords];   // blocks chosen by the tile's query blocks
  __shared__ int s_pre[kFuseWords];            // union entries in the words below
  const int ntiles = tile_count(D);
  const int per = D.B == 64 ? 2 : 1;                       // query blocks per tile
  const int nw = cdiv(NB, 32), nsink = D.S * D.nbpf;
  for (int p = 0; p < kFuseQb / per; ++p) {
    const int qa = qb0 + p * per;
    if (qa >= D.nqb) break;                                // the same for the whole CTA
    const int t = qa / per;
    const int nq = (per == 2 && qa + 1 < D.nqb) ? 2 : 1;
    for (int i = threadIdx.x; i < 2 * kFuseWords; i += blockDim.x) s_bits[i / kFuseWords][i % kFuseWords] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < nq * D.nsel; i += blockDim.x) {
      const int which = i / D.nsel;
      const int id = sl[(qa - qb0 + which) * D.nsel + i % D.nsel];   // < NB by construction
      atomicOr(&s_bits[which][id >> 5], 1u << (id & 31));
    }
    __syncthreads();
    if (warp == 0) {
      int carry = 0;
      for (int w0 = 0; w0 < nw; w0 += 32) {
        const int w = w0 + lane;
        const int own = w < nw ? __popc(s_bits[0][w] | s_bits[1][w]) : 0;
        int inc = own;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += v;
        }
        if (w < nw) s_pre[w] = carry + inc - own;
        carry += __shfl_sync(0xffffffffu, inc, 31);
      }
      if (lane == 0) plan_cnt[(size_t)h * ntiles + t] = nsink + carry;
    }
    __syncthreads();
    uint32_t* out = plan + ((size_t)h * ntiles + t) * plan_stride(D);
    for (int e = threadIdx.x; e < nsink; e += blockDim.x) out[e] = plan_pack(e / D.nbpf, e % D.nbpf, 3u);
    for (int x = threadIdx.x; x < NB; x += blockDim.x) {
      const int w = x >> 5;
      const uint32_t bit = 1u << (x & 31), ba = s_bits[0][w], bb = s_bits[1][w];
      if ((ba | bb) & bit) {
        const int pos = s_pre[w] + __popc((ba | bb) & (bit - 1u));
        out[nsink + pos] = plan_pack(D.S + x / D.nbpf, x % D.nbpf,
                                     ((ba & bit) ? 1u : 0u) | ((bb & bit) ? 2u : 0u));
      }
    }
    __syncthreads();                                       // the bitmaps are reused
  }
}

// Per (head, group of kFuseQb query blocks): frame scores by linearity from the block
// scores, frame top-k, block top-k in each chosen frame, block_idx, and the key plans of
// the group's query tiles.  A tile's plan is written by the whole CTA from two bitmaps
// over the F * n_bpf history blocks (one per query block of the tile): the union's bits
// in id order give the entries, a prefix count of the union's words their positions.
__global__ void __launch_bounds__(kPickThreads)
select_pick_kernel(const float* __restrict__ scores, int32_t* __restrict__ block_idx,
                   uint32_t* __restrict__ plan, int32_t* __restrict__ plan_cnt, const Dims D) {
  extern __shared__ float4 sm4[];
  pick_group(scores, block_idx, plan, plan_cnt, D, blockIdx.y, blockIdx.x * kFuseQb,
             reinterpret_cast<float*>(sm4));
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
