// lf_select.cuh — stages (a)-(c) of hierarchical sparse attention: token compression
// (mean pooling of query and key blocks, frame pooling) and the two-stage top-k
// selection of history frames and blocks.
//
// [LF-gist 2.2] "Light Forcing: Accelerating Autoregressive Video Diffusion via Sparse
// Attention" (gist.science explainer), section 2.2: queries and keys are compressed by
// mean pooling at block and frame granularity; each query block first retrieves a few
// history frames with the frame-level compressed keys, then the important blocks inside
// those frames with the block-level compressed keys.
// [LF-yly 三] the youleyou article, section 三: the same stages; similarity is an inner
// product.
#pragma once
#include "lf_common.cuh"

namespace lf {

// ---------------------------------------------------------------------------------
// (a) Pooling.  One CTA row (blockIdx.x) is one block of tokens: the first nqb rows are
// the current chunk's query blocks, the next F*nbpf rows the history key blocks, and (when
// the current chunk is sparse) the last nqb rows the current chunk's key blocks.  Each
// thread owns 8 consecutive channels of the H*d-wide token row (one 16-byte load per
// token), so a warp reads 512 contiguous bytes per token.  Sums are fp32 in a fixed
// order: four consecutive runs of the block's tokens, each in token order, then the runs
// in order.
// ---------------------------------------------------------------------------------
struct PoolArgs {
  const __nv_bfloat16* q;        // [ncur, H, d]
  const __nv_bfloat16* k_cache;  // [n_slots, T, H, d]
  float* q_blk;                  // [H, nqb, d]
  float* k_blk;                  // [H, F, nbpf, d]
  float* k_pool;                 // [n_slots, H, nbpf, d] pooled-key cache, or null: when
                                 // set, history blocks are written to their slot's rows
  const __nv_bfloat16* k_cur;    // [ncur, H, d] current-chunk keys (with kc_blk)
  float* kc_blk;                 // [H, nqb, d] current-chunk key block means, or null
  int hist_slots[LF_MAX_FRAMES];
};

constexpr int kPoolCols = 64;       // 8-channel groups per CTA (threads per token group)
constexpr int kPoolGroups = 4;      // token groups per CTA: a block's tokens split in 4 runs
constexpr int kPoolThreads = kPoolCols * kPoolGroups;
constexpr int kPoolUnroll = 8;     // 16-byte loads in flight per thread

// Thread (token group g, column group c): sums its run of the block's tokens in token order
// (16-byte loads, up to kPoolUnroll in flight; four CTAs per SM keep ~128 KB in flight per
// SM); the four runs are then added in run order.
__global__ void __launch_bounds__(kPoolThreads, 4)
pool_blocks_kernel(const __grid_constant__ PoolArgs a, const Dims D) {
  __shared__ float part[kPoolGroups][kPoolCols][8];
  const int unit = blockIdx.x;
  const int HD = D.H * D.d;
  const int col = threadIdx.x % kPoolCols, g = threadIdx.x / kPoolCols;
  const int vec = blockIdx.y * kPoolCols + col;               // 8-channel group
  const bool active = vec * 8 < HD;

  const __nv_bfloat16* base;
  int ntok;
  float* dst;
  const int h = (vec * 8) / D.d, c0 = (vec * 8) % D.d;
  const int hist_end = D.nqb + D.F * D.nbpf;
  if (unit < D.nqb || unit >= hist_end) {
    const bool is_q = unit < D.nqb;                 // query block, or current key block
    const int u = is_q ? unit : unit - hist_end;
    const int f = u / D.nbpf, b = u % D.nbpf;
    ntok = block_len(D, b);
    base = (is_q ? a.q : a.k_cur) + ((size_t)f * D.T + (size_t)b * D.B) * HD;
    dst = (is_q ? a.q_blk : a.kc_blk) + ((size_t)h * D.nqb + u) * D.d + c0;
  } else {
    const int u = unit - D.nqb;
    const int f = u / D.nbpf, b = u % D.nbpf;
    const int slot = a.hist_slots[f];
    ntok = block_len(D, b);
    base = a.k_cache + ((size_t)slot * D.T + (size_t)b * D.B) * HD;
    dst = a.k_pool != nullptr
        ? a.k_pool + (((size_t)slot * D.H + h) * D.nbpf + b) * D.d + c0
        : a.k_blk + (((size_t)h * D.F + f) * D.nbpf + b) * D.d + c0;
  }
  const int run = (ntok + kPoolGroups - 1) / kPoolGroups;
  const int t0 = g * run, t1 = min(ntok, t0 + run);
  const uint4* src = reinterpret_cast<const uint4*>(base) + vec;
  const size_t stride = HD / 8;     // uint4 per token row

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  if (active) {
    for (int t = t0; t < t1; t += kPoolUnroll) {
      uint4 v[kPoolUnroll];
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u)
        if (t + u < t1) v[u] = __ldg(src + (size_t)(t + u) * stride);
#pragma unroll
      for (int u = 0; u < kPoolUnroll; ++u) {
        if (t + u < t1) {
          const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v[u]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f2 = __bfloat1622float2(p[i]);
            acc[2 * i] += f2.x;
            acc[2 * i + 1] += f2.y;
          }
        }
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[g][col][i] = acc[i];
  __syncthreads();
  if (g != 0 || !active) return;
  float s[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    s[i] = ((part[0][col][i] + part[1][col][i]) + part[2][col][i]) + part[3][col][i];
  const float inv = 1.0f / (float)ntok;
  float4* o = reinterpret_cast<float4*>(dst);
  o[0] = make_float4(s[0] * inv, s[1] * inv, s[2] * inv, s[3] * inv);
  o[1] = make_float4(s[4] * inv, s[5] * inv, s[6] * inv, s[7] * inv);
}

// Frame pooling from the block means: k_frm = sum_b len_b * k_blk[b] / T (the frame mean
// over all T tokens, since block sums are len_b * mean_b).  One thread per channel.
__global__ void pool_frames_kernel(const float* __restrict__ k_blk, float* __restrict__ k_frm,
                                   const Dims D) {
  const int f = blockIdx.x, h = blockIdx.y;
  const float* src = k_blk + ((size_t)h * D.F + f) * D.nbpf * D.d;
  const float invT = 1.0f / (float)D.T;
  for (int c = threadIdx.x; c < D.d; c += blockDim.x) {
    float s = 0.f;
    for (int b0 = 0; b0 < D.nbpf; b0 += 32) {  // 32 loads in flight, summed in block order
      float v[32];
#pragma unroll
      for (int u = 0; u < 32; ++u)
        v[u] = b0 + u < D.nbpf ? src[(size_t)(b0 + u) * D.d + c] : 0.f;
#pragma unroll
      for (int u = 0; u < 32; ++u)
        if (b0 + u < D.nbpf) s += (float)block_len(D, b0 + u) * v[u];
    }
    k_frm[((size_t)h * D.F + f) * D.d + c] = s * invT;
  }
}

// ---------------------------------------------------------------------------------
// Warp top-k helpers.  Order: larger score first; equal scores -> lower index first.
// ---------------------------------------------------------------------------------
__device__ __forceinline__ bool better(float s1, int i1, float s2, int i2) {
  return s1 > s2 || (s1 == s2 && i1 < i2);
}

// Warp-wide argmax of (score, index) pairs with the order above; every lane gets it.
__device__ __forceinline__ void warp_argmax(float& s, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float so = __shfl_xor_sync(0xffffffffu, s, off);
    int io = __shfl_xor_sync(0xffffffffu, i, off);
    if (better(so, io, s, i)) { s = so; i = io; }
  }
}

constexpr int kMaxPerLane = 8;   // candidates per lane: up to 256 frames or blocks

// Selects the k best of n candidates held lane-strided (candidate c = lane + 32*j lives
// in sc[j] of lane c%32).  Returns in `taken` (bit j per lane) the chosen candidates.
// n <= 32: each lane counts the candidates better than its own (its rank) in one sweep
// of shuffles; larger n: k rounds of warp argmax.
__device__ __forceinline__ uint32_t warp_topk(const float* sc, int n, int k) {
  const int lane = threadIdx.x & 31;
  if (n <= 32) {
    int rank = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float sj = __shfl_sync(0xffffffffu, sc[0], j);
      rank += (j < n && better(sj, j, sc[0], lane)) ? 1 : 0;
    }
    return (lane < n && rank < k) ? 1u : 0u;
  }
  uint32_t taken = 0;
  for (int r = 0; r < k; ++r) {
    float bs = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
      const int c = lane + 32 * j;
      if (c < n && !((taken >> j) & 1u) && better(sc[j], c, bs, bi)) { bs = sc[j]; bi = c; }
    }
    warp_argmax(bs, bi);
    if (bi != 0x7fffffff && (bi & 31) == lane) taken |= 1u << (bi >> 5);
  }
  return taken;
}

// Writes the chosen candidate ids ascending: out[pos] = id_base + c.
__device__ __forceinline__ void warp_write_ascending(uint32_t taken, int n, int32_t* out,
                                                     int id_base) {
  const int lane = threadIdx.x & 31;
  int before = 0;
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    if (32 * j >= n) break;
    const uint32_t m = __ballot_sync(0xffffffffu, (taken >> j) & 1u);
    if ((taken >> j) & 1u) out[before + __popc(m & ((1u << lane) - 1u))] = id_base + lane + 32 * j;
    before += __popc(m);
  }
}

// q . k over d channels in a fixed order (four interleaved partial sums, then combined).
template <int HD>
__device__ __forceinline__ float dot_fixed(const float* q, const float* k) {
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
  for (int c = 0; c < HD; c += 4) {
    const float4 x = *reinterpret_cast<const float4*>(q + c);
    const float4 y = *reinterpret_cast<const float4*>(k + c);
    a0 = fmaf(x.x, y.x, a0); a1 = fmaf(x.y, y.y, a1); a2 = fmaf(x.z, y.z, a2); a3 = fmaf(x.w, y.w, a3);
  }
  return (a0 + a1) + (a2 + a3);
}

// ---------------------------------------------------------------------------------
// (b) Frame selection.  CTA = (group of 8 query blocks, head); k_frm[h] is staged in shared
// memory with a padded row pitch; warp w takes query block 8*blockIdx.x + w, lane c scores
// frames c, c+32, ... with a full-length dot product in fixed order.
// ---------------------------------------------------------------------------------
constexpr int kSelWarps = 8;

template <int HD>
__global__ void __launch_bounds__(kSelWarps * 32)
select_frames_kernel(const float* __restrict__ q_blk, const float* __restrict__ k_frm,
                     int32_t* __restrict__ frame_idx, float* __restrict__ frame_score,
                     const Dims D) {
  extern __shared__ float4 sm4[];
  float* sk = reinterpret_cast<float*>(sm4);
  const int h = blockIdx.y;
  const int pitch = D.d + 4;
  float* sq = sk + (size_t)D.F * pitch;               // [kSelWarps][d]
  for (int i = threadIdx.x; i < D.F * (D.d / 4); i += blockDim.x) {
    const int f = i / (D.d / 4), c4 = i % (D.d / 4);
    reinterpret_cast<float4*>(sk + (size_t)f * pitch)[c4] =
        reinterpret_cast<const float4*>(k_frm + ((size_t)h * D.F + f) * D.d)[c4];
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x * kSelWarps + warp;
  if (qb < D.nqb)
    for (int c4 = lane; c4 < D.d / 4; c4 += 32)
      reinterpret_cast<float4*>(sq + warp * D.d)[c4] =
          reinterpret_cast<const float4*>(q_blk + ((size_t)h * D.nqb + qb) * D.d)[c4];
  __syncthreads();
  if (qb >= D.nqb) return;

  float sc[kMaxPerLane];
  const float* qv = sq + warp * D.d;
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int f = lane + 32 * j;
    float s = -INFINITY;
    if (f < D.F) {
      s = dot_fixed<HD>(qv, sk + (size_t)f * pitch);
      if (frame_score) frame_score[((size_t)h * D.nqb + qb) * D.F + f] = s;
    }
    sc[j] = s;
  }
  const uint32_t taken = warp_topk(sc, D.F, D.kf);
  warp_write_ascending(taken, D.F, frame_idx + ((size_t)h * D.nqb + qb) * D.kf, 0);
}

// ---------------------------------------------------------------------------------
// Current-chunk block selection (sparse current chunk).  CTA = (group of 8 query blocks,
// head); kc_blk[h] is staged in shared memory with a padded row pitch; warp w takes query
// block qb = 8*blockIdx.x + w: lane c scores current blocks c, c+32, ... with a full-length
// dot product in fixed order, the own block qb gets +inf so that it is always kept, and the
// kc best are written ascending.
// ---------------------------------------------------------------------------------
template <int HD>
__global__ void __launch_bounds__(kSelWarps * 32)
select_current_kernel(const float* __restrict__ q_blk, const float* __restrict__ kc_blk,
                      int32_t* __restrict__ cur_idx, const Dims D) {
  extern __shared__ float4 sm4[];
  float* sk = reinterpret_cast<float*>(sm4);
  const int h = blockIdx.y;
  const int pitch = D.d + 4;
  float* sq = sk + (size_t)D.nqb * pitch;             // [kSelWarps][d]
  for (int i = threadIdx.x; i < D.nqb * (D.d / 4); i += blockDim.x) {
    const int c = i / (D.d / 4), c4 = i % (D.d / 4);
    reinterpret_cast<float4*>(sk + (size_t)c * pitch)[c4] =
        reinterpret_cast<const float4*>(kc_blk + ((size_t)h * D.nqb + c) * D.d)[c4];
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qb = blockIdx.x * kSelWarps + warp;
  if (qb < D.nqb)
    for (int c4 = lane; c4 < D.d / 4; c4 += 32)
      reinterpret_cast<float4*>(sq + warp * D.d)[c4] =
          reinterpret_cast<const float4*>(q_blk + ((size_t)h * D.nqb + qb) * D.d)[c4];
  __syncthreads();
  if (qb >= D.nqb) return;
  float sc[kMaxPerLane];
  const float* qv = sq + warp * D.d;
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int c = lane + 32 * j;
    float s = -INFINITY;
    if (c < D.nqb) s = c == qb ? INFINITY : dot_fixed<HD>(qv, sk + (size_t)c * pitch);
    sc[j] = s;
  }
  const uint32_t taken = warp_topk(sc, D.nqb, D.kc);
  warp_write_ascending(taken, D.nqb, cur_idx + ((size_t)h * D.nqb + qb) * D.kc, 0);
}

// ---------------------------------------------------------------------------------
// (c) Block selection inside chosen frames.  CTA = (history frame f, head h): k_blk[h, f]
// is staged in shared memory once, and the query blocks of head h whose chosen-frame list
// holds f (at rank j) are listed first; then, in batches whose pooled queries are staged
// in shared memory, a warp per query block scores the frame's blocks (lane c: blocks c,
// c+32, ...), keeps the kb best and writes them, ascending, to slots [j*kb, (j+1)*kb) of
// block_idx[h, qb] — ascending overall because the frame list is ascending.
// ---------------------------------------------------------------------------------
constexpr int kSelBatch = 32;
constexpr int kSelSplit = 4;      // CTAs per (frame, head): query blocks split in strides

template <int HD>
__global__ void __launch_bounds__(kSelWarps * 32)
select_blocks_kernel(const float* __restrict__ q_blk, const float* __restrict__ k_blk,
                     const int32_t* __restrict__ frame_idx, int32_t* __restrict__ block_idx,
                     float* __restrict__ block_score, const Dims D) {
  extern __shared__ float4 sm4[];
  float* sk = reinterpret_cast<float*>(sm4);
  const int f = blockIdx.x, h = blockIdx.y;
  const int pitch = D.d + 4;
  float* sq = sk + (size_t)D.nbpf * pitch;            // [kSelBatch][d]
  int* s_list = reinterpret_cast<int*>(sq + (size_t)kSelBatch * D.d);   // [nqb] packed qb | rank
  int* s_fl = s_list + D.nqb;                                             // [nqb * kf] frame lists
  __shared__ int s_n;
  if (threadIdx.x == 0) s_n = 0;
  for (int i = threadIdx.x; i < D.nbpf * (D.d / 4); i += blockDim.x) {
    const int b = i / (D.d / 4), c4 = i % (D.d / 4);
    reinterpret_cast<float4*>(sk + (size_t)b * pitch)[c4] =
        reinterpret_cast<const float4*>(k_blk + (((size_t)h * D.F + f) * D.nbpf + b) * D.d)[c4];
  }
  for (int i = threadIdx.x; i < D.nqb * D.kf; i += blockDim.x)
    s_fl[i] = frame_idx[(size_t)h * D.nqb * D.kf + i];
  __syncthreads();
  // which query blocks (of this CTA's stride) chose frame f, and at which rank (lists
  // validated on the way)
  for (int qb = blockIdx.z + threadIdx.x * kSelSplit; qb < D.nqb; qb += blockDim.x * kSelSplit) {
    const int* fl = s_fl + (size_t)qb * D.kf;
    int rank = -1;
    bool bad = false;
    int prev = -1;
    for (int j = 0; j < D.kf; ++j) {
      const int v = fl[j];
      bad |= v < 0 || v >= D.F || v <= prev;
      prev = v;
      if (v == f) rank = j;
    }
    if (bad) {
      if (f == 0 && blockIdx.z == 0) record_status(LF_ERR_BAD_INDEX);
    } else if (rank >= 0) {
      s_list[atomicAdd(&s_n, 1)] = (qb << 10) | rank;
    }
  }
  __syncthreads();
  const int n = s_n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int b0 = 0; b0 < n; b0 += kSelBatch) {
    const int nb = min(kSelBatch, n - b0);
    for (int i = threadIdx.x; i < nb * (D.d / 4); i += blockDim.x) {
      const int e = i / (D.d / 4), c4 = i % (D.d / 4);
      const int qb = s_list[b0 + e] >> 10;
      reinterpret_cast<float4*>(sq + (size_t)e * D.d)[c4] =
          reinterpret_cast<const float4*>(q_blk + ((size_t)h * D.nqb + qb) * D.d)[c4];
    }
    __syncthreads();
    for (int e = warp; e < nb; e += kSelWarps) {
      const int qb = s_list[b0 + e] >> 10, rank = s_list[b0 + e] & 1023;
      const float* qv = sq + (size_t)e * D.d;
      float sc[kMaxPerLane];
#pragma unroll
      for (int j = 0; j < kMaxPerLane; ++j) {
        const int b = lane + 32 * j;
        float sres = -INFINITY;
        if (b < D.nbpf) {
          sres = dot_fixed<HD>(qv, sk + (size_t)b * pitch);
          if (block_score)
            block_score[(((size_t)h * D.nqb + qb) * D.kf + rank) * D.nbpf + b] = sres;
        }
        sc[j] = sres;
      }
      const uint32_t taken = warp_topk(sc, D.nbpf, D.kb);
      warp_write_ascending(taken, D.nbpf,
                           block_idx + ((size_t)h * D.nqb + qb) * D.nsel + (size_t)rank * D.kb,
                           f * D.nbpf);
    }
    __syncthreads();
  }
}

}  // namespace lf
