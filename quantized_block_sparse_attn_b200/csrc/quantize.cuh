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
//
// Both quantisers are bound by HBM bandwidth.  Algorithmic bytes: the bf16 input read
// once, the 8-bit codes and the fp32 scales written once (V's column maxima need the whole
// sequence before the first code, so V is read twice; see below).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"

namespace qbsa {

constexpr int kQuantThreads = 256;

// bf16 magnitudes of 8 packed values (4 words) -> running max per 16-bit lane.  For
// non-negative bf16 bit patterns the integer order is the value order.
__device__ __forceinline__ void amax_bf16x8(const uint4& u, uint32_t (&m)[4]) {
  m[0] = __vmaxu2(m[0], u.x & 0x7fff7fffu);
  m[1] = __vmaxu2(m[1], u.y & 0x7fff7fffu);
  m[2] = __vmaxu2(m[2], u.z & 0x7fff7fffu);
  m[3] = __vmaxu2(m[3], u.w & 0x7fff7fffu);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Codes of x / s taken in IEEE float32 division (round to nearest) without dividing in the
// common case.  With r = RN(1/s) and y = RN(x * r), |y - x/s| <= 2^-23 |x/s|, and RN(x/s)
// is within 2^-24 |x/s| of x/s, so both lie between y (1 - 2^-20) and y (1 + 2^-20) (each
// product rounded once more, still inside).  Rounding to an integer or to E4M3 is monotone:
// if both ends of that bracket give the same code, every value between them does, the
// correctly rounded quotient included.  Otherwise (a quotient within about 2^-20 of a code
// boundary, roughly one value in 10^4 to 10^5) the quotient is divided exactly.
constexpr float kBracketLo = 1.0f - 9.5367431640625e-07f;  // 1 - 2^-20
constexpr float kBracketHi = 1.0f + 9.5367431640625e-07f;  // 1 + 2^-20

// r = RN(1 / s) for the bracket, or 0 when 1 / s overflows (a subnormal s): every code of
// that scale then takes the exact division (a zero r never passes the bracket test below,
// whose two ends agree only through a finite, correctly bracketed product)
__device__ __forceinline__ float bracket_recip(float s) {
  const float r = __frcp_rn(s);
  return (r <= 3.0e38f) ? r : 0.0f;
}

// INT8 code of RN(x / s) as the low byte of a 32-bit word, with r = bracket_recip(s).
// fma(y, 1 -/+ 2^-20, 1.5 * 2^23) rounds the exact bracket end to an integer (|y| < 2^22 puts
// the sum in [2^23, 2^24), where the float spacing is 1; round to nearest, ties to even), and
// the sum's low byte is that integer's two's-complement byte.  |x / s| <= 127 (1 + 2^-24)
// because s = RN(max|x| / 127), so the integer never leaves [-127, 127] and needs no clamp.
__device__ __forceinline__ uint32_t int8_code_byte(float x, float s, float r) {
  const float y = x * r;
  const float lo = __fmaf_rn(y, kBracketLo, 12582912.0f), hi = __fmaf_rn(y, kBracketHi, 12582912.0f);
  if (lo == hi && r != 0.0f) return __float_as_uint(lo);
  return static_cast<uint32_t>(__float2int_rn(__fdiv_rn(x, s)));
}

// Two E4M3 codes (byte 0 = x0) of RN(x0 / s0), RN(x1 / s1), nearest even, saturating;
// r0, r1 from bracket_recip
__device__ __forceinline__ uint32_t e4m3x2_code(float x0, float s0, float r0, float x1, float s1, float r1) {
  const float y0 = x0 * r0, y1 = x1 * r1;
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(y1 * kBracketLo), "f"(y0 * kBracketLo));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(y1 * kBracketHi), "f"(y0 * kBracketHi));
  if (lo == hi && r0 != 0.0f && r1 != 0.0f) return lo;
  uint16_t ex;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(ex) : "f"(__fdiv_rn(x1, s1)), "f"(__fdiv_rn(x0, s0)));
  return ex;
}

// 16-byte read of input that no kernel writes while this one runs: no L1 allocation, and (no
// volatile) free for the compiler to issue every load of a thread before the first use
__device__ __forceinline__ uint4 ld_stream_v4(const uint4* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

// The low bytes of b0..b3 packed into one word (byte i = b_i).
__device__ __forceinline__ uint32_t pack_low_bytes(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// -------------------------------------------------------------------------------------
// Q / K: per-128-row-block INT8
// -------------------------------------------------------------------------------------

// One CTA per (block, head, batch), 256 threads; x is BNSD [B, N, S, D] bf16.  The block
// (128 rows x D) is read once into registers with 16-byte loads: its maximum magnitude,
// then the codes from the same registers.
template <int D>
__global__ void __launch_bounds__(kQuantThreads) quantize_qk_kernel(const __nv_bfloat16* __restrict__ x, int N, int S,
                                                                     int8_t* __restrict__ codes,
                                                                     float* __restrict__ scales) {
  constexpr int kChunksPerRow = D / 8;
  constexpr int kPerThread = 128 * kChunksPerRow / kQuantThreads;
  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int rows = min(128, S - kb * 128);
  const int64_t base = (((int64_t)b * N + h) * S + (int64_t)kb * 128) * D;
  const uint4* src = reinterpret_cast<const uint4*>(x + base);
  const int n_chunks = rows * kChunksPerRow;

  uint4 r[kPerThread];
  uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = threadIdx.x + k * kQuantThreads;
    r[k] = i < n_chunks ? ld_stream_v4(src + i) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) amax_bf16x8(r[k], m);
  const uint32_t mm = __vmaxu2(__vmaxu2(m[0], m[1]), __vmaxu2(m[2], m[3]));
  uint32_t a_bits = max(mm & 0xffffu, mm >> 16) << 16;  // float bits of the larger bf16 magnitude
  a_bits = __reduce_max_sync(0xffffffffu, a_bits);
  __shared__ uint32_t red[kQuantThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a_bits;
  __syncthreads();
  uint32_t v = 0u;
#pragma unroll
  for (int w = 0; w < kQuantThreads / 32; ++w) v = max(v, red[w]);
  const float a = __uint_as_float(v);
  const float s = (a == 0.f) ? 1.0f : __fdiv_rn(a, 127.0f);
  const float rs = bracket_recip(s);

  uint2* dst = reinterpret_cast<uint2*>(codes + base);
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = threadIdx.x + k * kQuantThreads;
    if (i < n_chunks) {
      float f[8];
      bf16x8_to_f32(r[k], f);
      uint32_t c[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) c[e] = int8_code_byte(f[e], s, rs);
      dst[i] = make_uint2(pack_low_bytes(c[0], c[1], c[2], c[3]), pack_low_bytes(c[4], c[5], c[6], c[7]));
    }
  }
  if (threadIdx.x == 0) scales[((int64_t)b * N + h) * gridDim.x + kb] = s;
}

// -------------------------------------------------------------------------------------
// V: per-channel E4M3 in two streaming passes
// -------------------------------------------------------------------------------------
//
// Each (b, h) "head" of V is cut into chunks of kRows rows, one CTA per (head, chunk):
//   v_colmax_kernel: the chunk's column maxima (16-byte loads, packed 16-bit integer max),
//                    folded into the head's maxima (scratch, zeroed first) with atomicMax;
//   v_quant_kernel:  the scales s_c = amax / 448 and the chunk's E4M3 codes; the chunk-0 CTA
//                    of each head writes the scales.
// The kernel boundary orders every maximum before any code.  DRAM traffic: V read twice (the
// second pass finds next to nothing of the first pass's data in L2: 0.13 % L2 hits measured at
// S = 65536), codes written once.

template <int D>
struct VQuantCfg {
  static constexpr int kTPR = D / 8;                   // threads per row, 8 channels each
  static constexpr int kRPI = kQuantThreads / kTPR;    // rows per iteration of the CTA
  static constexpr int kIters = 8;
  static constexpr int kRows = kRPI * kIters;          // rows per chunk (128 at D = 128: 32 KB)
};

struct VQuantParams {
  const __nv_bfloat16* v;
  uint8_t* codes;
  float* scales;
  unsigned int* amax;     // scratch, [H, D] float bits, zero before the first pass
  int H;
  int S;
  int n_ch;               // chunks per head
};

template <int D>
__global__ void __launch_bounds__(kQuantThreads) v_colmax_kernel(VQuantParams p) {
  using C = VQuantCfg<D>;
  __shared__ uint32_t s_red[kQuantThreads / 32][D / 2];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = tid % C::kTPR;  // channels [8 cg, 8 cg + 8)
  const int ri = tid / C::kTPR;  // row within an iteration
  const int g = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.n_ch));
  const int c = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.n_ch));
  const int r0 = c * C::kRows;
  const int rows = min(C::kRows, p.S - r0);
  const uint4* src = reinterpret_cast<const uint4*>(p.v + ((int64_t)g * p.S + r0) * D) + cg;
  uint4 u[C::kIters];
#pragma unroll
  for (int k = 0; k < C::kIters; ++k) {
    const int row = ri + k * C::kRPI;
    u[k] = row < rows ? ld_stream_v4(src + (int64_t)row * C::kTPR) : make_uint4(0u, 0u, 0u, 0u);
  }
  uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int k = 0; k < C::kIters; ++k) amax_bf16x8(u[k], m);
#pragma unroll
  for (int o = C::kTPR; o < 32; o <<= 1) {
#pragma unroll
    for (int j = 0; j < 4; ++j) m[j] = __vmaxu2(m[j], __shfl_xor_sync(0xffffffffu, m[j], o));
  }
  if (lane < C::kTPR) {
#pragma unroll
    for (int j = 0; j < 4; ++j) s_red[warp][cg * 4 + j] = m[j];
  }
  __syncthreads();
  if (tid < D / 2) {
    uint32_t mm = 0u;
#pragma unroll
    for (int w = 0; w < kQuantThreads / 32; ++w) mm = __vmaxu2(mm, s_red[w][tid]);
    unsigned int* am = p.amax + (int64_t)g * D + 2 * tid;
    atomicMax(am, (mm & 0xffffu) << 16);
    atomicMax(am + 1, mm & 0xffff0000u);
  }
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads, 3) v_quant_kernel(VQuantParams p) {
  using C = VQuantCfg<D>;
  const int tid = threadIdx.x;
  const int cg = tid % C::kTPR;
  const int ri = tid / C::kTPR;
  const int g = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.n_ch));
  const int c = static_cast<int>(blockIdx.x % static_cast<unsigned>(p.n_ch));
  const int r0 = c * C::kRows;
  const int rows = min(C::kRows, p.S - r0);
  const int64_t row0 = (int64_t)g * p.S + r0;
  const uint4* src = reinterpret_cast<const uint4*>(p.v + row0 * D) + cg;
  uint4 u[C::kIters];
#pragma unroll
  for (int k = 0; k < C::kIters; ++k) {
    const int row = ri + k * C::kRPI;
    u[k] = row < rows ? ld_stream_v4(src + (int64_t)row * C::kTPR) : make_uint4(0u, 0u, 0u, 0u);
  }
  float s[8], rs[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float a = __uint_as_float(__ldg(p.amax + (int64_t)g * D + cg * 8 + j));
    s[j] = (a == 0.f) ? 1.0f : __fdiv_rn(a, 448.0f);
    rs[j] = bracket_recip(s[j]);
  }
  if (c == 0 && ri == 0) {
    float4* sc = reinterpret_cast<float4*>(p.scales + (int64_t)g * D + cg * 8);
    sc[0] = make_float4(s[0], s[1], s[2], s[3]);
    sc[1] = make_float4(s[4], s[5], s[6], s[7]);
  }
  uint2* dst = reinterpret_cast<uint2*>(p.codes + row0 * D) + cg;
#pragma unroll
  for (int k = 0; k < C::kIters; ++k) {
    const int row = ri + k * C::kRPI;
    if (row < rows) {
      float f[8];
      bf16x8_to_f32(u[k], f);
      uint32_t w[2];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t pr = e4m3x2_code(f[2 * e], s[2 * e], rs[2 * e], f[2 * e + 1], s[2 * e + 1], rs[2 * e + 1]);
        if ((e & 1) == 0) w[e >> 1] = pr;
        else w[e >> 1] |= pr << 16;
      }
      dst[(int64_t)row * C::kTPR] = make_uint2(w[0], w[1]);
    }
  }
}

}  // namespace qbsa
