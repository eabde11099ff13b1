// Block-mask estimation for block-sparse attention: block mean pooling and per-query-block
// top-k of the pooled scores.
//
// EagleQBSA article ("昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍"),
// section "背景介绍": block-sparse attention (AdaBSA) computes only the 128x128 blocks a
// block mask selects; section "MindIE SD调用方式" passes the mask as block_sparse_mask
// with block_shape=[128,128].  The article does not describe how the mask is chosen; this
// file implements the plain reading: mean-pool each 128-token block of Q and K, score a
// block pair by scale * <q_mean, k_mean> (the block's average logit), keep the n_keep
// best key blocks per query block, equal scores to the lower block index.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "schedule.cuh"

namespace qbsa {

constexpr int kEstThreads = 128;
constexpr int kTopkThreads = 256;
constexpr int kTopkMaxKBlocks = 2048;

// One CTA per (b, n, 128-token block): x bf16 [B, N, S, D] -> mean [B, N, ceil(S/128), D] fp32.
// Each thread reads 16-byte chunks (8 channels) of every (128 / (D / 8))-th row; the row
// groups are then summed in shared memory.  D in {64, 128, 256}.
__global__ void __launch_bounds__(kEstThreads) block_mean_kernel(const __nv_bfloat16* __restrict__ x, int S, int D,
                                                                 int nb, float* __restrict__ out) {
  __shared__ float part[kEstThreads * 8];
  const int blk = blockIdx.x % nb;
  const int64_t bn = blockIdx.x / nb;
  const int lanes_per_row = D / 8;
  const int rows_per_iter = kEstThreads / lanes_per_row;
  const int c8 = threadIdx.x % lanes_per_row;
  const int rg = threadIdx.x / lanes_per_row;
  const int r0 = blk * kTile, r1 = min(S, r0 + kTile);
  const __nv_bfloat16* base = x + bn * S * D;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  for (int r = r0 + rg; r < r1; r += rows_per_iter) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(base + (int64_t)r * D) + c8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += __uint_as_float(w[i] << 16);              // bf16 -> f32 is a shift
      acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) part[rg * D + c8 * 8 + i] = acc[i];
  __syncthreads();
  const float inv = 1.0f / static_cast<float>(r1 - r0);
  for (int d = threadIdx.x; d < D; d += kEstThreads) {
    float s = 0.f;
    for (int g = 0; g < rows_per_iter; ++g) s += part[g * D + d];
    out[(bn * nb + blk) * D + d] = s * inv;
  }
}

// Orderable score key: unsigned order equals the order of the scores (-0 taken as +0).
__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t u = __float_as_uint(s + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Query blocks per CTA of block_topk_kernel: the pooled key matrix of a head is read once per
// group of this many query blocks.
constexpr int kTopkGroup = 8;
__host__ inline int topk_smem_bytes(int nkb, int D) { return kTopkGroup * (D + nkb) * 4; }

// One CTA per (b, h, group of kTopkGroup query blocks).
// Phase 1: thread j' owns key rows j = j' + 256 k and scores each against every pooled query of
//          the group (the queries sit in shared memory and are read as broadcasts).
// Phase 2: warp u selects for query block u: the n_keep-th largest score key v is found bit by
//          bit (32 counting passes), every key > v is kept, and the remaining places go to the
//          keys equal to v in ascending block order; the mask row is written (1 = compute).
__global__ void __launch_bounds__(kTopkThreads) block_topk_kernel(const float* __restrict__ qm,
                                                                  const float* __restrict__ km, int Nq, int group,
                                                                  int nqb, int nkb, int D, float scale, int n_keep,
                                                                  uint8_t* __restrict__ mask,
                                                                  float* __restrict__ scores) {
  extern __shared__ __align__(16) uint8_t topk_smem[];
  float* qrows = reinterpret_cast<float*>(topk_smem);                              // [group][D]
  uint32_t* keys = reinterpret_cast<uint32_t*>(topk_smem + kTopkGroup * D * 4);    // [group][nkb]
  const int n_grp = (nqb + kTopkGroup - 1) / kTopkGroup;
  const int i0 = (blockIdx.x % n_grp) * kTopkGroup;
  const int nq = min(kTopkGroup, nqb - i0);
  const int64_t bh = blockIdx.x / n_grp;  // b * Nq + h
  const int h = static_cast<int>(bh % Nq);
  const int64_t b = bh / Nq;
  const int64_t bg = b * (Nq / group) + h / group;
  for (int e = threadIdx.x; e < kTopkGroup * D; e += kTopkThreads) {
    const int u = e / D;
    qrows[e] = (u < nq) ? qm[(bh * nqb + i0 + u) * D + (e - u * D)] : 0.f;
  }
  __syncthreads();
  const float* kbase = km + bg * nkb * D;
  const int d4n = D >> 2;
  for (int j = threadIdx.x; j < nkb; j += kTopkThreads) {
    const float4* krow = reinterpret_cast<const float4*>(kbase + (int64_t)j * D);
    float s[kTopkGroup];
#pragma unroll
    for (int u = 0; u < kTopkGroup; ++u) s[u] = 0.f;
    for (int d4 = 0; d4 < d4n; ++d4) {
      const float4 kv = __ldg(krow + d4);
#pragma unroll
      for (int u = 0; u < kTopkGroup; ++u) {
        const float4 qv = reinterpret_cast<const float4*>(qrows + u * D)[d4];
        s[u] = fmaf(qv.w, kv.w, fmaf(qv.z, kv.z, fmaf(qv.y, kv.y, fmaf(qv.x, kv.x, s[u]))));
      }
    }
#pragma unroll
    for (int u = 0; u < kTopkGroup; ++u) {
      if (u < nq) {
        const float sc = s[u] * scale;
        keys[u * nkb + j] = score_key(sc);
        if (scores) scores[(bh * nqb + i0 + u) * nkb + j] = sc;
      }
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int u = warp; u < nq; u += kTopkThreads / 32) {
    const uint32_t* kr = keys + u * nkb;
    // largest v with #{key >= v} >= n_keep, one bit at a time from the top
    uint32_t v = 0;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = v | (1u << bit);
      int c = 0;
      for (int j = lane; j < nkb; j += 32) c += (kr[j] >= cand) ? 1 : 0;
      c = __reduce_add_sync(0xffffffffu, c);
      if (c >= n_keep) v = cand;
    }
    int above = 0;
    for (int j = lane; j < nkb; j += 32) above += (kr[j] > v) ? 1 : 0;
    above = __reduce_add_sync(0xffffffffu, above);
    int ties_left = n_keep - above;  // keys equal to v still to keep, lowest block index first
    uint8_t* mrow = mask + (bh * nqb + i0 + u) * nkb;
    for (int j0 = 0; j0 < nkb; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = (j < nkb) ? kr[j] : 0u;
      const bool tie = (j < nkb) && key == v;
      const uint32_t tb = __ballot_sync(0xffffffffu, tie);
      const int before = __popc(tb & ((1u << lane) - 1u));
      const bool keep = (j < nkb) && (key > v || (tie && before < ties_left));
      if (j < nkb) mrow[j] = keep ? 1 : 0;
      ties_left -= __popc(tb);
    }
  }
}

}  // namespace qbsa
