// On-GPU quantisers that prepare qbsa_fwd's inputs from bf16 Q, K, V.
//
// EagleQBSA article ("昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍",
// section "EagleQBSA量化叠加稀疏方案设计", Fig 2.1): Q and K use symmetric linear INT8
// with one scale per 128-token block of the sequence axis; V uses FP8 E4M3 with one
// scale per channel (head-dim column) over the whole sequence.  The article does not
// spell out the scale rule; this library takes a = max|x| (float32), s = a/127 (INT8)
// or a/448 (E4M3), s = 1 when a = 0, codes rint_half_even(x/s) clamped to ±127, and
// E4M3 codes x/s rounded to nearest even with saturation.  Divisions are IEEE
// round-to-nearest so results are reproducible bit for bit.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace qbsa {

// One CTA per (block, head, batch); 256 threads; x is BNSD [B, N, S, D] bf16.
__global__ void quantize_qk_kernel(const __nv_bfloat16* __restrict__ x, int N, int S, int D,
                                   int8_t* __restrict__ codes, float* __restrict__ scales) {
  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int nblk = gridDim.x;
  const int r0 = kb * 128;
  const int rows = min(128, S - r0);
  const int64_t base = (((int64_t)b * N + h) * S + r0) * D;
  const int n = rows * D;
  float a = 0.f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) a = fmaxf(a, fabsf(__bfloat162float(x[base + i])));
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  __shared__ float red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  a = red[0];
  const float s = (a == 0.f) ? 1.0f : __fdiv_rn(a, 127.0f);
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    int q = __float2int_rn(__fdiv_rn(__bfloat162float(x[base + i]), s));
    q = max(-127, min(127, q));
    codes[base + i] = static_cast<int8_t>(q);
  }
  if (threadIdx.x == 0) scales[((int64_t)b * N + h) * nblk + kb] = s;
}

// Column max |v| over the sequence, into amax_bits (float bits; >= 0 so integer max
// orders them).  Grid (row chunks, heads, batch), blockDim.x == D.
__global__ void v_colmax_kernel(const __nv_bfloat16* __restrict__ v, int N, int S, int D, int rows_per_cta,
                                unsigned int* __restrict__ amax_bits) {
  const int c = threadIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int r0 = blockIdx.x * rows_per_cta;
  const int r1 = min(S, r0 + rows_per_cta);
  const int64_t base = ((int64_t)b * N + h) * S * D;
  float a = 0.f;
  for (int r = r0; r < r1; ++r) a = fmaxf(a, fabsf(__bfloat162float(v[base + (int64_t)r * D + c])));
  atomicMax(&amax_bits[((int64_t)b * N + h) * D + c], __float_as_uint(a));
}

__global__ void v_scale_kernel(float* __restrict__ scales, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    const float a = scales[i];  // holds max|v| on entry
    scales[i] = (a == 0.f) ? 1.0f : __fdiv_rn(a, 448.0f);
  }
}

// E4M3 codes of v / s_c; grid-stride over [B*N*S*D / 2] pairs.
__global__ void v_quant_kernel(const __nv_bfloat16* __restrict__ v, int N, int S, int D,
                               const float* __restrict__ scales, uint8_t* __restrict__ codes, int64_t total) {
  for (int64_t i = (int64_t)(blockIdx.x * blockDim.x + threadIdx.x) * 2; i < total;
       i += (int64_t)gridDim.x * blockDim.x * 2) {
    const int c = static_cast<int>(i % D);
    const int64_t bh = i / ((int64_t)S * D);
    const float s0 = scales[bh * D + c], s1 = scales[bh * D + c + 1];
    const float x0 = __fdiv_rn(__bfloat162float(v[i]), s0);
    const float x1 = __fdiv_rn(__bfloat162float(v[i + 1]), s1);
    uint16_t pr;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(x1), "f"(x0));
    *reinterpret_cast<uint16_t*>(codes + i) = pr;
  }
}

}  // namespace qbsa
