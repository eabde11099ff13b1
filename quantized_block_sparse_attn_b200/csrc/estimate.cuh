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

// Orderable 64-bit sort key: ascending key = descending score, then ascending index.
__device__ __forceinline__ uint64_t topk_key(float s, int j) {
  const uint32_t u = __float_as_uint(s);
  const uint32_t up = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending with the score
  return (static_cast<uint64_t>(~up) << 32) | static_cast<uint32_t>(j);
}

// One CTA per (b, h, query block): scores of all key blocks of kv head h / group, a bitonic
// sort of the (score, index) keys in shared memory, and the mask row (1 = compute).
__global__ void __launch_bounds__(kTopkThreads) block_topk_kernel(const float* __restrict__ qm,
                                                                  const float* __restrict__ km, int Nq, int group,
                                                                  int nqb, int nkb, int D, float scale, int n_keep,
                                                                  uint8_t* __restrict__ mask,
                                                                  float* __restrict__ scores) {
  __shared__ uint64_t keys[kTopkMaxKBlocks];
  __shared__ uint8_t sel[kTopkMaxKBlocks];
  __shared__ float qrow[1024];
  const int i = blockIdx.x % nqb;
  const int64_t bh = blockIdx.x / nqb;  // b * Nq + h
  const int h = static_cast<int>(bh % Nq);
  const int64_t b = bh / Nq;
  const int64_t bg = b * (Nq / group) + h / group;
  for (int d = threadIdx.x; d < D; d += kTopkThreads) qrow[d] = qm[(bh * nqb + i) * D + d];
  int npow = 1;
  while (npow < nkb) npow <<= 1;
  for (int j = threadIdx.x; j < npow; j += kTopkThreads) {
    keys[j] = ~0ull;  // padding sorts last
    if (j < nkb) sel[j] = 0;
  }
  __syncthreads();
  // warp-cooperative dot products: lanes split the channels, a shuffle tree sums them
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* kbase = km + bg * nkb * D;
  for (int j = warp; j < nkb; j += kTopkThreads / 32) {
    float s = 0.f;
    for (int d = lane; d < D; d += 32) s = fmaf(qrow[d], kbase[(int64_t)j * D + d], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    s *= scale;
    if (lane == 0) {
      keys[j] = topk_key(s, j);
      if (scores) scores[(bh * nqb + i) * nkb + j] = s;
    }
  }
  __syncthreads();
  // bitonic sort, ascending, over npow keys
  for (int k = 2; k <= npow; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int t = threadIdx.x; t < npow; t += kTopkThreads) {
        const int p = t ^ jj;
        if (p > t) {
          const uint64_t a = keys[t], c = keys[p];
          const bool up = (t & k) == 0;
          if ((a > c) == up) {
            keys[t] = c;
            keys[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int r = threadIdx.x; r < n_keep; r += kTopkThreads) sel[static_cast<uint32_t>(keys[r])] = 1;
  __syncthreads();
  uint8_t* mrow = mask + (bh * nqb + i) * nkb;
  for (int j = threadIdx.x; j < nkb; j += kTopkThreads) mrow[j] = sel[j];
}

}  // namespace qbsa
