// Quantized block-sparse attention forward (EagleQBSA) for sm_100a.
//
// EagleQBSA article ("昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍"):
// Q and K arrive as INT8 with one scale per 128-token block, V as FP8 E4M3 with one
// scale per channel, and P is rounded to FP8 before P·V (section
// "EagleQBSA量化叠加稀疏方案设计", Fig 2.1); only the 128x128 blocks selected by the
// block-sparse mask are computed (section "背景介绍"; block_sparse_mask and
// block_shape=[128,128] in section "MindIE SD调用方式").
//
// One CTA per (batch, head, 128-row query block).  Warp 0 first compacts the CTA's row
// of the block mask into the ascending list of kept key blocks in shared memory, with
// each block's dequantisation constant s_q * s_k * scale * log2(e).  Then:
//   warp 0      TMA producer (Q once; K and V tiles of kept blocks, 3-stage rings)
//   warp 1      TMEM owner + MMA issuer: S = Q8 K8ᵀ (kind::i8, s32 in TMEM);
//               O += P8 V8 (kind::f8f6f4, A = P8 from TMEM, B = V8 MN-major) and
//               L += P8 · 1 (N = 16 ones matrix), so L is exactly Σ p8.
//   warps 2..9  softmax: query row 32*(warp%4)+lane; warps 2..5 own key columns [0,64),
//               warps 6..9 [64,128), exchanging partial row maxima through shared
//               memory.  Exact s32 -> f32 (|dot| < 2^24), online softmax whose weights
//               p = 2^(z - R) use a power-of-two reference R re-set to ceil(running max)
//               only when the max exceeds it by more than 8 (exact power-of-two
//               rescales of O and L, rare), P -> E4M3 into TMEM, epilogue
//               O * v_scale / L -> bf16.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) L [384,400) P0 [448,480) P1 [480,512).
//
// CTA order: query heads in groups whose K8/V8 fit in about 48 MB of L2, query blocks
// in order, heads fastest inside a group.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"

namespace qbsa {

constexpr int kQbsaMaxKBlocks = 2048;  // key blocks per row of the mask (S_kv <= 256K)

struct QbsaParams {
  CUtensorMap tm_q;  // 4-D {128, rows, heads, batch} int8, box {128, 128, 1, 1}, SW128
  CUtensorMap tm_k;
  CUtensorMap tm_v;  // E4M3 bytes, same geometry
  const float* q_scale;   // [B, Nq, nqb]
  const float* k_scale;   // [B, Nkv, nkb]
  const float* v_scale;   // [B, Nkv, 128]
  const uint8_t* block_mask;  // [B, Nq, nqb, nkb], 1 = compute
  __nv_bfloat16* out;     // [B, Nq, Sq, 128]
  float* softmax_max;     // [B, Nq, Sq] or nullptr
  float* softmax_sum;
  int B, Nq, Nkv, Sq, Skv, group, nqb, nkb;
  int n_rank;             // B * nqb
  int head_grp;           // query heads per L2 group
  float scale_log2;       // scale * log2(e)
};

struct QbsaCfg {
  static constexpr int D = 128;
  static constexpr int kStages = 3;
  static constexpr int kTileBytes = kTile * 128;  // 128 rows x 128 bytes
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kOnesOff = kVOff + kStages * kTileBytes;  // 16 x 128 bytes of E4M3 1.0
  static constexpr int kCOff = kOnesOff + 2048;                   // float dequant constant per kept block
  static constexpr int kListOff = kCOff + kQbsaMaxKBlocks * 4;    // uint16 kept-block list
  static constexpr int kXOff = kListOff + kQbsaMaxKBlocks * 2;    // int row-max exchange [2][2][128]
  static constexpr int kBarOff = kXOff + 2 * 2 * 128 * 4;
  static constexpr int kBarQFull = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kStages;
  static constexpr int kBarVFull = kBarKEmpty + kStages;
  static constexpr int kBarVEmpty = kBarVFull + kStages;
  static constexpr int kBarSFull = kBarVEmpty + kStages;
  static constexpr int kBarSFree = kBarSFull + 2;
  static constexpr int kBarPFull = kBarSFree + 2;
  static constexpr int kBarPVDone = kBarPFull + 2;
  static constexpr int kBarOFinal = kBarPVDone + 1;  // last P·V done (single use)
  static constexpr int kNumBars = kBarOFinal + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem addr, abort flag, list count
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColL = 384, kColP0 = 448, kColP1 = 480;
  static constexpr int kThreads = 320;
  static constexpr int kSoftmaxThreads = 256;
};

// Compact one row of the block mask (n_kb bytes, 1 = keep) into ascending indices.
// Executed by one full warp; returns the count (same value in every lane).
__device__ __forceinline__ int compact_mask_row(const uint8_t* row, int n_kb, uint16_t* list, int lane) {
  int count = 0;
  for (int base = 0; base < n_kb; base += 32) {
    const int j = base + lane;
    const bool keep = (j < n_kb) && (row[j] != 0);
    const uint32_t m = __ballot_sync(0xffffffffu, keep);
    if (keep) list[count + __popc(m & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
    count += __popc(m);
  }
  return count;
}

__device__ __forceinline__ void qbsa_named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__global__ void __launch_bounds__(320, 1) attn_qbsa_kernel(const __grid_constant__ QbsaParams p) {
  using C = QbsaCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_base = smem_u32(smem_raw);
  const uint32_t base = (raw_base + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_base);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t bar0 = base + C::kBarOff;
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);
  int* count_slot = reinterpret_cast<int*>(smem + C::kMiscOff + 8);
  uint16_t* list = reinterpret_cast<uint16_t*>(smem + C::kListOff);
  float* cst_list = reinterpret_cast<float*>(smem + C::kCOff);
  float* xch = reinterpret_cast<float*>(smem + C::kXOff);

  // head groups (L2 reuse of K/V), query blocks in order, heads fastest inside a group
  const int64_t per_group = (int64_t)p.head_grp * p.n_rank;
  const int grp = static_cast<int>(blockIdx.x / per_group);
  const int h0 = grp * p.head_grp;
  const int hcount = min(p.head_grp, p.Nq - h0);
  const int off = static_cast<int>(blockIdx.x - grp * per_group);
  const int r = off / hcount;
  const int h = h0 + off % hcount;
  const int qb = r % p.nqb;
  const int b = r / p.nqb;
  const int g = h / p.group;

  if (warp == 0) {
    const uint8_t* mrow = p.block_mask + (((int64_t)b * p.Nq + h) * p.nqb + qb) * p.nkb;
    const int cnt = compact_mask_row(mrow, p.nkb, list, lane);
    __syncwarp();
    const float sq = p.q_scale[((int64_t)b * p.Nq + h) * p.nqb + qb];
    const float* ks = p.k_scale + ((int64_t)b * p.Nkv + g) * p.nkb;
    for (int i = lane; i < cnt; i += 32) cst_list[i] = (sq * ks[list[i]]) * p.scale_log2;
    if (lane == 0) {
      *count_slot = cnt;
      *abort_flag = 0;
      mbar_init(bar(C::kBarQFull), 1);
      for (int s = 0; s < C::kStages; ++s) {
        mbar_init(bar(C::kBarKFull + s), 1);
        mbar_init(bar(C::kBarKEmpty + s), 1);
        mbar_init(bar(C::kBarVFull + s), 1);
        mbar_init(bar(C::kBarVEmpty + s), 1);
      }
      for (int b2 = 0; b2 < 2; ++b2) {
        mbar_init(bar(C::kBarSFull + b2), 1);
        mbar_init(bar(C::kBarSFree + b2), C::kSoftmaxThreads);
        mbar_init(bar(C::kBarPFull + b2), C::kSoftmaxThreads);
      }
      mbar_init(bar(C::kBarPVDone), 1);
      mbar_init(bar(C::kBarOFinal), 1);
      fence_mbar_init();
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  } else if (warp == 2) {
    // the ones matrix (E4M3 1.0 = 0x38) used to accumulate the row sums of P8
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::kOnesOff);
    for (int i = lane; i < 512; i += 32) ones[i] = 0x38383838u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n = *count_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && n > 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      mbar_arrive_expect_tx(bar(C::kBarQFull), C::kTileBytes);
      tma_load_4d(base + C::kQOff, &p.tm_q, bar(C::kBarQFull), 0, qb * kTile, h, b, pol_q);
      for (int it = 0; it < n; ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        const int kv_row = static_cast<int>(list[it]) * kTile;
        if (it >= C::kStages && !mbar_wait(bar(C::kBarKEmpty + s), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::kBarKFull + s), C::kTileBytes);
        tma_load_4d(base + C::kKOff + s * C::kTileBytes, &p.tm_k, bar(C::kBarKFull + s), 0, kv_row, g, b, pol_kv);
        if (it >= C::kStages && !mbar_wait(bar(C::kBarVEmpty + s), ph ^ 1, abort_flag)) break;
        mbar_arrive_expect_tx(bar(C::kBarVFull + s), C::kTileBytes);
        tma_load_4d(base + C::kVOff + s * C::kTileBytes, &p.tm_v, bar(C::kBarVFull + s), 0, kv_row, g, b, pol_kv);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_s8(128, 128);
      constexpr uint32_t idesc_pv = idesc_e4m3(128, 128, true);
      constexpr uint32_t idesc_pl = idesc_e4m3(128, 16, false);
      const uint32_t ones = base + C::kOnesOff;
      bool ok = mbar_wait(bar(C::kBarQFull), 0, abort_flag);
      auto issue_pv = [&](int j) -> bool {
        const int bj = j & 1;
        const int s = j % C::kStages;
        if (!mbar_wait(bar(C::kBarPFull + bj), (j >> 1) & 1, abort_flag)) return false;
        if (!mbar_wait(bar(C::kBarVFull + s), (j / C::kStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vbase = base + C::kVOff + s * C::kTileBytes;
        const uint32_t pcol = bj ? C::kColP1 : C::kColP0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // 32 key rows per step: 8 TMEM columns of packed P8, 4096 B of V8
          const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
          mma_f8_ts(tmem + C::kColO, tmem + pcol + kk * 8, sdesc_sw128(vbase + kk * 4096, C::kTileBytes, 1024),
                    idesc_pv, acc);
          mma_f8_ts(tmem + C::kColL, tmem + pcol + kk * 8, sdesc_sw128(ones + kk * 32, 16, 1024), idesc_pl, acc);
        }
        mma_commit(bar(C::kBarPVDone));
        mma_commit(bar(C::kBarVEmpty + s));
        return true;
      };
      const uint32_t qbase = base + C::kQOff;
      for (int it = 0; ok && it < n; ++it) {
        const int s = it % C::kStages;
        const int bi = it & 1;
        if (!mbar_wait(bar(C::kBarKFull + s), (it / C::kStages) & 1, abort_flag)) { ok = false; break; }
        if (it >= 2 && !mbar_wait(bar(C::kBarSFree + bi), ((it - 2) >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kbase = base + C::kKOff + s * C::kTileBytes;
        const uint32_t scol = bi ? C::kColS1 : C::kColS0;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_i8_ss(tmem + scol, sdesc_sw128(qbase + kk * 32, 16, 1024), sdesc_sw128(kbase + kk * 32, 16, 1024),
                    idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(C::kBarSFull + bi));
        mma_commit(bar(C::kBarKEmpty + s));
        if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
      }
      if (ok && issue_pv(n - 1)) mma_commit(bar(C::kBarOFinal));
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // 0: key columns [0,64), 1: [64,128)
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t i_glob = (int64_t)qb * kTile + row;
    const float kNegInf = -__int_as_float(0x7f800000);
    const uint32_t o_col = tmem + lane_off + C::kColO + half * 64;
    const uint32_t l_col = tmem + lane_off + C::kColL;

    float m = kNegInf;    // running max, log2 domain
    float ref = kNegInf;  // power-of-two reference of the FP8 weights (an integer)
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int kb = list[it];
      const int bi = it & 1;
      const float cst = cst_list[it];
      const int valid = min(kTile, p.Skv - kb * kTile) - half * 64;  // valid columns of this half
      // never leave the loop early (the paired warp waits on named barriers below)
      if (ok) ok = mbar_wait(bar(C::kBarSFull + bi), (it >> 1) & 1, abort_flag);
      tc_fence_after();
      float sv[64];  // exact: |dot| <= 128 * 127^2 < 2^24
      {
        uint32_t r[64];
        tmem_ld64_wait(tmem + lane_off + (bi ? C::kColS1 : C::kColS0) + half * 64, r);
#pragma unroll
        for (int x = 0; x < 64; ++x) sv[x] = __int2float_rn(static_cast<int32_t>(r[x]));
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarSFree + bi));

      if (valid < 64) {  // tail block: keys past S_kv get -inf (p = 0 below)
#pragma unroll
        for (int x = 0; x < 64; ++x)
          if (x >= valid) sv[x] = kNegInf;
      }
      const float pmax = max64(sv);
      float* slot = xch + (it & 1) * 256;
      slot[half * 128 + row] = pmax;
      qbsa_named_bar_sync(1 + quarter, 64);
      const float tmax = fmaxf(pmax, slot[(half ^ 1) * 128 + row]);

      // max(t) * c == max(t * c): multiplication by c > 0 is monotone in float
      const float m_blk = tmax * cst;
      m = fmaxf(m, m_blk);
      // power-of-two reference: re-set to ceil(m) once m exceeds it by more than 8, so
      // p <= 2^8 stays below E4M3's 448 and every rescale is an exact power of two
      const bool upd = (ref == kNegInf) || (m > ref + 8.0f);
      const float new_ref = upd ? ceilf(m) : ref;
      const bool need = upd && (ref != kNegInf);
      // 2^(ref - new_ref) built from its exponent bits (exact; flush below 2^-126)
      const int dexp = need ? static_cast<int>(ref - new_ref) : 0;
      const float a = (dexp < -126) ? 0.f : __int_as_float((127 + dexp) << 23);
      ref = new_ref;
      if (__any_sync(0xffffffffu, need)) {
        if (ok) ok = mbar_wait(bar(C::kBarPVDone), (it - 1) & 1, abort_flag);
        tc_fence_after();
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          tmem_ld32_wait(o_col + ch * 32, r);
#pragma unroll
          for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * a);
          tmem_st32(o_col + ch * 32, r);
        }
        if (half == 0) tmem_st1(l_col, __float_as_uint(__uint_as_float(tmem_ld1_wait(l_col)) * a));
        tmem_st_wait();
      }
      // p = 2^(t c - R) held in FP16 (the precision of P before its FP8 rounding),
      // two weights per ex2, then rounded to E4M3
      uint32_t pk[16];
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        pk[x] = exp2_e4m3x4(fmaf(sv[4 * x], cst, -ref), fmaf(sv[4 * x + 1], cst, -ref),
                            fmaf(sv[4 * x + 2], cst, -ref), fmaf(sv[4 * x + 3], cst, -ref));
      }
      tmem_st16(tmem + lane_off + (bi ? C::kColP1 : C::kColP0) + half * 16, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + bi));
    }

    // ------------------------------------------------------------ epilogue
    const bool row_valid = i_glob < p.Sq;
    bool have_o = ok && n > 0;
    if (have_o) {
      // a dedicated single-use barrier: pv_done's parity cannot tell PV(n-1) from PV(n-3)
      have_o = mbar_wait(bar(C::kBarOFinal), 0, abort_flag);
      tc_fence_after();
    }
    float l = 0.f;
    if (have_o) l = __uint_as_float(tmem_ld1_wait(l_col));
    const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
    const float* vsc = p.v_scale + ((int64_t)b * p.Nkv + g) * 128 + half * 64;
    __nv_bfloat16* orow = p.out + (((int64_t)b * p.Nq + h) * p.Sq + i_glob) * 128 + half * 64;
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      uint32_t r[32];
      if (have_o) {
        tmem_ld32_wait(o_col + ch * 32, r);
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) r[x] = 0u;
      }
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          float f[8];
#pragma unroll
          for (int y = 0; y < 8; ++y) f[y] = __uint_as_float(r[8 * x + y]) * (vsc[ch * 32 + 8 * x + y] * inv_l);
          uint4 v;
          v.x = pack_bf16x2(f[0], f[1]);
          v.y = pack_bf16x2(f[2], f[3]);
          v.z = pack_bf16x2(f[4], f[5]);
          v.w = pack_bf16x2(f[6], f[7]);
          dst[x] = v;
        }
      }
    }
    if (half == 0 && row_valid) {
      const int64_t sidx = ((int64_t)b * p.Nq + h) * p.Sq + i_glob;
      const bool live = l > 0.f;
      if (p.softmax_max) p.softmax_max[sidx] = live ? m * 0.6931471805599453f : kNegInf;
      if (p.softmax_sum) p.softmax_sum[sidx] = live ? l * ex2(ref - m) : 0.f;  // against the true max
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Test hook: run the CTA-side mask compaction for every mask row (one warp per row).
__global__ void qbsa_block_lists_kernel(const uint8_t* mask, int rows, int n_kb, int32_t* lists, int32_t* counts) {
  __shared__ uint16_t buf[4][kQbsaMaxKBlocks];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.x * 4 + warp;
  if (r >= rows) return;
  const int cnt = compact_mask_row(mask + (int64_t)r * n_kb, n_kb, buf[warp], lane);
  __syncwarp();
  for (int i = lane; i < n_kb; i += 32) lists[(int64_t)r * n_kb + i] = (i < cnt) ? buf[warp][i] : -1;
  if (lane == 0) counts[r] = cnt;
}

}  // namespace qbsa
