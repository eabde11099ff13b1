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
// once, the 8-bit codes and the fp32 scales written once.
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

__device__ __forceinline__ uint4 ld_stream_v4(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
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

  uint2* dst = reinterpret_cast<uint2*>(codes + base);
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = threadIdx.x + k * kQuantThreads;
    if (i < n_chunks) {
      float f[8];
      bf16x8_to_f32(r[k], f);
      uint32_t w[2] = {0u, 0u};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int q = max(-127, min(127, __float2int_rn(__fdiv_rn(f[e], s))));
        w[e >> 2] |= (static_cast<uint32_t>(q) & 0xffu) << (8 * (e & 3));
      }
      dst[i] = make_uint2(w[0], w[1]);
    }
  }
  if (threadIdx.x == 0) scales[((int64_t)b * N + h) * gridDim.x + kb] = s;
}

// -------------------------------------------------------------------------------------
// V: per-channel E4M3, one pass over HBM
// -------------------------------------------------------------------------------------
//
// Each (b, h) "head" of V is cut into chunks of kRows rows.  Work items are
//   pass 1 (g, c): the column maxima of chunk c of head g, folded into the head's maxima
//                  with atomicMax, then one arrival on the head's counter;
//   pass 2 (g, c): once all chunks of head g have arrived, the scales s_c = amax/448 and
//                  the E4M3 codes of chunk c.
// Persistent CTAs take items in ticket order from an atomic counter: pass 1 of head 0,
// then pass 1 of head g + 1 alternating chunk by chunk with pass 2 of head g, then pass 2
// of the last head.  Every pass-1 item of a head is handed out before any pass-2 item of
// that head, so a pass-2 item only waits for items already running, and the chunk it
// re-reads was read from HBM about two heads earlier, so it is still in L2 while heads
// are at most ~40 MB (S = 128K at D = 128 is 32 MB).  DRAM traffic is one read of V and
// one write of the codes.
//
// Scratch (zeroed before the launch): ticket counter, one arrival counter per head, the
// per-head column maxima as float bits.

template <int D>
struct VQuantCfg {
  static constexpr int kTPR = D / 8;                   // threads per row, 8 channels each
  static constexpr int kRPI = kQuantThreads / kTPR;    // rows per iteration of the CTA
  static constexpr int kIters = 16;
  static constexpr int kRows = kRPI * kIters;          // rows per work item (256 at D = 128)
};

struct VQuantParams {
  const __nv_bfloat16* v;
  uint8_t* codes;
  float* scales;
  unsigned int* ticket;   // scratch
  unsigned int* arrived;  // scratch, [H]
  unsigned int* amax;     // scratch, [H, D] float bits
  int H;
  int S;
  int n_ch;
  unsigned int total;     // 2 * H * n_ch
};

// Waits (bounded) until *ctr >= target; acquire ordering on success.
__device__ __forceinline__ bool wait_count_at_least(const unsigned int* ctr, unsigned int target) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= target) return true;
    __nanosleep(100);
    if ((it & 15u) == 15u && global_timer_ns() - t0 > QBSA_WAIT_TIMEOUT_NS) {
      atomicCAS(&g_device_error, 0u, static_cast<unsigned int>(kErrTimeout));
      return false;
    }
  }
}

// ticket -> (pass, head, chunk) in the order described above
__device__ __forceinline__ void v_item(unsigned int t, int H, int n_ch, int& pass, int& g, int& c) {
  const unsigned int n = static_cast<unsigned int>(n_ch);
  const unsigned int mid = 2u * n * static_cast<unsigned int>(H - 1);
  if (t < n) {
    pass = 1; g = 0; c = static_cast<int>(t);
  } else if (t >= n + mid) {
    pass = 2; g = H - 1; c = static_cast<int>(t - n - mid);
  } else {
    const unsigned int u = t - n;
    const unsigned int w = u / (2u * n), r = u % (2u * n);
    c = static_cast<int>(r >> 1);
    if ((r & 1u) == 0u) {
      pass = 1; g = static_cast<int>(w) + 1;
    } else {
      pass = 2; g = static_cast<int>(w);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kQuantThreads) v_quant_kernel(VQuantParams p) {
  using C = VQuantCfg<D>;
  __shared__ unsigned int s_ticket;
  __shared__ int s_ok;
  __shared__ uint32_t s_red[kQuantThreads / 32][D / 2];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int cg = tid % C::kTPR;  // channels [8 cg, 8 cg + 8)
  const int ri = tid / C::kTPR;  // row within an iteration
  if (tid == 0) s_ticket = atomicAdd(p.ticket, 1u);
  __syncthreads();
  unsigned int t = s_ticket;
  while (t < p.total) {
    int pass, g, c;
    v_item(t, p.H, p.n_ch, pass, g, c);
    __syncthreads();                                    // every thread has read s_ticket
    if (tid == 0) s_ticket = atomicAdd(p.ticket, 1u);   // the next item, fetched while this one runs
    const int r0 = c * C::kRows;
    const int rows = min(C::kRows, p.S - r0);
    const int64_t row0 = (int64_t)g * p.S + r0;
    const uint4* src = reinterpret_cast<const uint4*>(p.v + row0 * D) + cg;
    if (pass == 1) {
      uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int k = 0; k < C::kIters; ++k) {
        const int row = ri + k * C::kRPI;
        if (row < rows) amax_bf16x8(__ldg(src + (int64_t)row * C::kTPR), m);
      }
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
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        atomicAdd(p.arrived + g, 1u);
      }
    } else {
      if (tid == 0) s_ok = wait_count_at_least(p.arrived + g, static_cast<unsigned int>(p.n_ch)) ? 1 : 0;
      __syncthreads();
      if (s_ok) {
        float s[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float a = __uint_as_float(__ldcg(p.amax + (int64_t)g * D + cg * 8 + j));
          s[j] = (a == 0.f) ? 1.0f : __fdiv_rn(a, 448.0f);
        }
        if (c == 0 && ri == 0) {
          float4* sc = reinterpret_cast<float4*>(p.scales + (int64_t)g * D + cg * 8);
          sc[0] = make_float4(s[0], s[1], s[2], s[3]);
          sc[1] = make_float4(s[4], s[5], s[6], s[7]);
        }
        uint2* dst = reinterpret_cast<uint2*>(p.codes + row0 * D) + cg;
#pragma unroll 4
        for (int k = 0; k < C::kIters; ++k) {
          const int row = ri + k * C::kRPI;
          if (row < rows) {
            float f[8];
            bf16x8_to_f32(__ldg(src + (int64_t)row * C::kTPR), f);
            uint32_t w[2];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint16_t pr;
              const float x0 = __fdiv_rn(f[2 * e], s[2 * e]);
              const float x1 = __fdiv_rn(f[2 * e + 1], s[2 * e + 1]);
              asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(x1), "f"(x0));
              if ((e & 1) == 0) w[e >> 1] = pr;
              else w[e >> 1] |= static_cast<uint32_t>(pr) << 16;
            }
            dst[(int64_t)row * C::kTPR] = make_uint2(w[0], w[1]);
          }
        }
      }
    }
    __syncthreads();  // s_ticket holds the next item; s_red and s_ok are free again
    t = s_ticket;
  }
}

}  // namespace qbsa
