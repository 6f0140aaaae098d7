// lf_fused.cuh — stages (b) and (c) fused, with the attention key plans, for the
// one-call path (lf_forward_chunk).
//
// Per (head, group of kFuseQb query blocks): the scores of every history block against
// the group's pooled queries (a small GEMM, q_blk[8 x d] . k_blk[F*n_bpf x d]^T, fixed
// summation order), the frame scores from them by linearity (a frame's pooled key is the
// length-weighted mean of its block keys, so its score is the length-weighted mean of
// the block scores), the top-k_f frames, the top-k_b blocks in each chosen frame, and the
// key plans of the group's query tiles.  [LF-gist 2.2] two-stage mask selection;
// [LF-yly 三] inner-product similarity.
#pragma once
#include "lf_select.cuh"
#include "lf_attn.cuh"

namespace lf {

constexpr int kFuseQb = 8;                 // query blocks per CTA (even: whole tile pairs)
constexpr int kFuseMaxBlocks = 2048;       // F * n_bpf handled by the fused path
constexpr int kFuseMaxSel = 256;           // k_f * k_b handled by the fused path

__host__ __device__ inline bool fused_select_ok(const Dims& D) {
  return D.F > 0 && D.F * D.nbpf <= kFuseMaxBlocks && D.nsel <= kFuseMaxSel &&
         D.F <= 32 * kMaxPerLane && D.nbpf <= 32 * kMaxPerLane;
}

__host__ __device__ inline size_t fused_select_smem(const Dims& D) {
  return (size_t)kFuseQb * D.d * 4 + (size_t)kFuseQb * D.F * D.nbpf * 4 +
         (size_t)kFuseQb * D.nsel * 4 + (size_t)kFuseQb * D.kf * 4;
}

template <int HD>
__global__ void __launch_bounds__(256)
select_fused_kernel(const float* __restrict__ q_blk, const float* __restrict__ k_blk,
                    int32_t* __restrict__ block_idx, uint32_t* __restrict__ plan,
                    int32_t* __restrict__ plan_cnt, const Dims D) {
  extern __shared__ float4 sm4[];
  float* sq = reinterpret_cast<float*>(sm4);                       // [kFuseQb][HD]
  const int NB = D.F * D.nbpf;
  float* sc = sq + kFuseQb * HD;                                    // [kFuseQb][NB]
  int32_t* sl = reinterpret_cast<int32_t*>(sc + (size_t)kFuseQb * NB);   // [kFuseQb][nsel]
  int32_t* sf = sl + kFuseQb * D.nsel;                              // [kFuseQb][kf]
  const int h = blockIdx.y, qb0 = blockIdx.x * kFuseQb;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < kFuseQb * (HD / 4); i += blockDim.x) {
    const int g = i / (HD / 4), c4 = i % (HD / 4);
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (qb0 + g < D.nqb)
      v = reinterpret_cast<const float4*>(q_blk + ((size_t)h * D.nqb + qb0 + g) * HD)[c4];
    reinterpret_cast<float4*>(sq + g * HD)[c4] = v;
  }
  __syncthreads();

  // block scores: thread t takes rows t, t + 256, ... of k_blk[h] (two at a time); each
  // score is one fixed-order sum over the channels
  const float* kh = k_blk + (size_t)h * NB * HD;
  for (int r0 = threadIdx.x; r0 < NB; r0 += 2 * blockDim.x) {
    const int r1 = r0 + blockDim.x;
    const bool has1 = r1 < NB;
    float acc0[kFuseQb], acc1[kFuseQb];
#pragma unroll
    for (int g = 0; g < kFuseQb; ++g) acc0[g] = acc1[g] = 0.f;
    const float4* k0 = reinterpret_cast<const float4*>(kh + (size_t)r0 * HD);
    const float4* k1 = reinterpret_cast<const float4*>(kh + (size_t)(has1 ? r1 : r0) * HD);
#pragma unroll 4
    for (int c4 = 0; c4 < HD / 4; ++c4) {
      const float4 a = __ldg(k0 + c4);
      const float4 b = __ldg(k1 + c4);
#pragma unroll
      for (int g = 0; g < kFuseQb; ++g) {
        const float4 q = reinterpret_cast<const float4*>(sq + g * HD)[c4];
        acc0[g] = fmaf(q.x, a.x, acc0[g]); acc0[g] = fmaf(q.y, a.y, acc0[g]);
        acc0[g] = fmaf(q.z, a.z, acc0[g]); acc0[g] = fmaf(q.w, a.w, acc0[g]);
        acc1[g] = fmaf(q.x, b.x, acc1[g]); acc1[g] = fmaf(q.y, b.y, acc1[g]);
        acc1[g] = fmaf(q.z, b.z, acc1[g]); acc1[g] = fmaf(q.w, b.w, acc1[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < kFuseQb; ++g) {
      sc[(size_t)g * NB + r0] = acc0[g];
      if (has1) sc[(size_t)g * NB + r1] = acc1[g];
    }
  }
  __syncthreads();

  // per query block (warp g): frame scores, frame top-k, block top-k in chosen frames
  const float invT = 1.0f / (float)D.T;
  for (int g = warp; g < kFuseQb; g += blockDim.x / 32) {
    const int qb = qb0 + g;
    if (qb >= D.nqb) continue;
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
    __syncwarp();
    for (int j = 0; j < D.kf; ++j) {
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
    __syncwarp();
    int32_t* dst = block_idx + ((size_t)h * D.nqb + qb) * D.nsel;
    for (int i = lane; i < D.nsel; i += 32) dst[i] = sl[g * D.nsel + i];
  }
  __syncthreads();

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

}  // namespace lf
