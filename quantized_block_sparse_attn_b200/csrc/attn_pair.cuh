// Dense bf16 fused attention forward for sm_100a, two query tiles per CTA.
//
// Computes Softmax(Q·Kᵀ·scale)·V (npu_fusion_attention guide, "昇腾 NPU 融合注意力算子详解与
// 迁移指南", §2 算子数学原理) for the unmasked case (no atten_mask, no pse, sparse_mode 0
// with a band that covers every pair), D = 128, BNSD or BSND, with the same online
// softmax and outputs (§5: attention_out, softmax_max, softmax_sum) as attn_dense_kernel,
// which serves every other case.
//
// One CTA owns two adjacent 128-row query tiles of one (batch, head).  Both tiles walk
// the same K/V tiles, so each K/V tile is loaded once for two tiles, and the two tiles
// take turns on one TMEM score buffer: while one tile's softmax warps turn scores into
// probabilities on the special-function unit, the tensor core computes the other tile's
// scores and the previous probabilities' P·V.
//
// CTA = 11 warps:
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1: query row 32*(warp%4)+lane (the warp's
//                    TMEM lane quarter), all 128 key columns of a block; O is rescaled in
//                    TMEM only when the running max grew by more than 2^8 (the lagging
//                    reference cancels in O / l; the statistics are corrected at the end);
//                    P goes to TMEM as bf16; the epilogue normalises O, stages it in the
//                    tile's Q buffer and writes it with TMA stores.
//   warp 8           TMA producer: both Q tiles once, then K and V tiles into rings.
//   warp 9           TMEM owner + QK issuer: S = Q_t·K_jᵀ (kind::f16, both operands from
//                    shared memory), tile 0 then tile 1 for every key tile j.
//   warp 10          P·V issuer: O_t += P_t·V_j (kind::f16, A = P_t from TMEM, B = V_j from
//                    shared memory, MN-major); each P·V is queued behind the same tile's
//                    next QK, which is on the softmax warps' critical path.
// TMEM columns: O0 [0,128) O1 [128,256) S [256,384) P0 [384,448) P1 [448,512).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "schedule.cuh"

namespace qbsa {

struct PairParams {
  CUtensorMap tm_q;  // 4-D {128, rows, heads, batch}, box {64, 128, 1, 1}, bf16, SW128
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_o;  // the output, same layout and box as tm_q
  float* softmax_max;  // [B, Nq, Sq] or nullptr
  float* softmax_sum;
  int B, Nq, Nkv, Sq, Skv, group;
  int n_qtiles;  // ceil(Sq / 128)
  int n_ktiles;  // ceil(Skv / 128)
  int n_pair;    // ceil(n_qtiles / 2)
  int n_rank;    // B * n_pair
  int head_grp;  // query heads per L2 group
  float scale;
};

struct PairCfg {
  static constexpr int D = 128;
  static constexpr int kKStages = 3;
  static constexpr int kVStages = 2;
  static constexpr int kTileBytes = kTile * D * 2;  // one 128 x 128 bf16 tile = two swizzle columns
  static constexpr int kSubBytes = kTile * 128;     // one 128-row x 128-byte swizzle column
  static constexpr int kQOff = 0;                   // Q of tile 0, then tile 1 (later: output staging)
  static constexpr int kKOff = kQOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kBarQFull = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kKStages;
  static constexpr int kBarVFull = kBarKEmpty + kKStages;
  static constexpr int kBarVEmpty = kBarVFull + kVStages;
  static constexpr int kBarSFull = kBarVEmpty + kVStages;  // [2], per tile
  static constexpr int kBarSFree = kBarSFull + 2;          // [2], per tile
  static constexpr int kBarPFull = kBarSFree + 2;          // [2]
  static constexpr int kBarPVDone = kBarPFull + 2;         // [2]
  static constexpr int kBarOFinal = kBarPVDone + 2;        // [2], single use
  static constexpr int kBarDrain = kBarOFinal + 2;         // [2] single use: every MMA of an issuer retired
  static constexpr int kNumBars = kBarDrain + 2;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem addr, abort flag, qk_issued[2]
  static constexpr int kSmemBytes = kMiscOff + 32 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO0 = 0, kColO1 = 128, kColS = 256, kColP = 384;  // P_t at kColP + 64 t
  static constexpr int kThreads = 352;
  static constexpr int kWarpProducer = 8, kWarpQK = 9, kWarpPV = 10;
};
static_assert(PairCfg::kSmemBytes <= 232448, "shared memory above the 227 KB opt-in limit");
static_assert(PairCfg::kKOff % 1024 == 0 && PairCfg::kVOff % 1024 == 0 && PairCfg::kTileBytes % 1024 == 0,
              "swizzled buffers must start on 1024-byte boundaries");

// acc += (a, b) on two packed f32 lanes (add.rn.f32x2: one instruction per pair of scores).
__device__ __forceinline__ void add_f32x2(uint64_t& acc, float a, float b) {
  asm("{\n\t.reg .b64 q;\n\tmov.b64 q, {%1, %2};\n\tadd.rn.f32x2 %0, %0, q;\n\t}" : "+l"(acc) : "f"(a), "f"(b));
}
// Sum of the two f32 lanes of a packed pair.
__device__ __forceinline__ float sum_f32x2(uint64_t v) {
  float a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
  return a + b;
}

__global__ void __launch_bounds__(352, 1) attn_pair_kernel(const __grid_constant__ PairParams p) {
  using C = PairCfg;
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
  volatile int* qk_issued = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 16);  // [2] QKs issued per tile

  // head groups (L2 reuse of K/V), query-tile pairs in order, heads fastest in a group
  const int64_t per_group = (int64_t)p.head_grp * p.n_rank;
  const int grp = static_cast<int>(blockIdx.x / per_group);
  const int h0 = grp * p.head_grp;
  const int hcount = min(p.head_grp, p.Nq - h0);
  const int off = static_cast<int>(blockIdx.x - grp * per_group);
  const int r = off / hcount;
  const int h = h0 + off % hcount;
  const int pr = r % p.n_pair;
  const int b = r / p.n_pair;
  const int g = h / p.group;
  const bool has1 = 2 * pr + 1 < p.n_qtiles;  // the second tile exists
  const int n = p.n_ktiles;                   // key tiles visited by each tile
  const int ntile = has1 ? 2 : 1;

  if (warp == C::kWarpProducer) {
    if (lane == 0) {
      *abort_flag = 0;
      qk_issued[0] = 0;
      qk_issued[1] = 0;
      mbar_init(bar(C::kBarQFull), 1);
      for (int s = 0; s < C::kKStages; ++s) {
        mbar_init(bar(C::kBarKFull + s), 1);
        mbar_init(bar(C::kBarKEmpty + s), 1);
      }
      for (int s = 0; s < C::kVStages; ++s) {
        mbar_init(bar(C::kBarVFull + s), 1);
        mbar_init(bar(C::kBarVEmpty + s), 1);
      }
      for (int t = 0; t < 2; ++t) {
        mbar_init(bar(C::kBarSFull + t), 1);
        mbar_init(bar(C::kBarSFree + t), 4);  // one arrival per softmax warp of the tile
        mbar_init(bar(C::kBarPFull + t), 4);
        mbar_init(bar(C::kBarPVDone + t), 1);
        mbar_init(bar(C::kBarOFinal + t), 1);
        mbar_init(bar(C::kBarDrain + t), 1);
      }
      fence_mbar_init();
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
      tma_prefetch_desc(&p.tm_o);
    }
  } else if (warp == C::kWarpQK) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == C::kWarpProducer) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && n > 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      mbar_arrive_expect_tx(bar(C::kBarQFull), C::kTileBytes * ntile);
      for (int t = 0; t < ntile; ++t)
        for (int sub = 0; sub < 2; ++sub)
          tma_load_4d(base + C::kQOff + t * C::kTileBytes + sub * C::kSubBytes, &p.tm_q, bar(C::kBarQFull),
                      sub * 64, (2 * pr + t) * kTile, h, b, pol_q);
      int kq = 0, vq = 0;  // K / V copies issued
      for (int j = 0; j < n; ++j) {
        const int kv_row = j * kTile;
        const int sk = j % C::kKStages, sv = j % C::kVStages;
        if (j >= C::kKStages &&
            !mbar_wait(bar(C::kBarKEmpty + sk), (static_cast<uint32_t>(j / C::kKStages) & 1) ^ 1, abort_flag))
          break;
        mbar_arrive_expect_tx(bar(C::kBarKFull + sk), C::kTileBytes);
        for (int sub = 0; sub < 2; ++sub)
          tma_load_4d(base + C::kKOff + sk * C::kTileBytes + sub * C::kSubBytes, &p.tm_k, bar(C::kBarKFull + sk),
                      sub * 64, kv_row, g, b, pol_kv);
        ++kq;
        if (j >= C::kVStages &&
            !mbar_wait(bar(C::kBarVEmpty + sv), (static_cast<uint32_t>(j / C::kVStages) & 1) ^ 1, abort_flag))
          break;
        mbar_arrive_expect_tx(bar(C::kBarVFull + sv), C::kTileBytes);
        for (int sub = 0; sub < 2; ++sub)
          tma_load_4d(base + C::kVOff + sv * C::kTileBytes + sub * C::kSubBytes, &p.tm_v, bar(C::kBarVFull + sv),
                      sub * 64, kv_row, g, b, pol_kv);
        ++vq;
      }
      // let the copies still in flight land before the CTA can exit (matters only after an
      // abort): an older copy's stage was reused, so it had been consumed
      for (int q = max(0, kq - C::kKStages); q < kq; ++q)
        mbar_wait_drain(bar(C::kBarKFull + q % C::kKStages), static_cast<uint32_t>(q / C::kKStages) & 1);
      for (int q = max(0, vq - C::kVStages); q < vq; ++q)
        mbar_wait_drain(bar(C::kBarVFull + q % C::kVStages), static_cast<uint32_t>(q / C::kVStages) & 1);
      mbar_wait_drain(bar(C::kBarQFull), 0);
    }
  } else if (warp == C::kWarpQK) {
    // ---------------------------------------------------------------- QK issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false);
      bool ok = mbar_wait(bar(C::kBarQFull), 0, abort_flag);
      int prev_t = -1, prev_j = 0;  // reader of the S buffer's current contents
      for (int j = 0; ok && j < n; ++j) {
        const int s = j % C::kKStages;
        if (!mbar_wait(bar(C::kBarKFull + s), static_cast<uint32_t>(j / C::kKStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t kbase = base + C::kKOff + s * C::kTileBytes;
        for (int t = 0; ok && t < ntile; ++t) {
          if (prev_t >= 0 && !mbar_wait(bar(C::kBarSFree + prev_t), static_cast<uint32_t>(prev_j) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qbase = base + C::kQOff + t * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // 16 elements (32 bytes) per step inside a 64-wide swizzle column
            const uint32_t o = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
            mma_f16_ss(tmem + C::kColS, sdesc_sw128(qbase + o, 16, 1024), sdesc_sw128(kbase + o, 16, 1024), idesc_qk,
                       kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::kBarSFull + t));
          if (t == ntile - 1) mma_commit(bar(C::kBarKEmpty + s));  // both tiles' QKs of K_j retired
          qk_issued[t] = j + 1;  // lets the PV issuer queue behind this QK
          prev_t = t;
          prev_j = j;
        }
      }
      // every MMA issued above has retired before TMEM can be released
      mma_commit(bar(C::kBarDrain));
      mbar_wait_drain(bar(C::kBarDrain), 0);
    }
  } else if (warp == C::kWarpPV) {
    // ---------------------------------------------------------------- PV issuer
    if (lane == 0 && n > 0) {
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, true);
      bool ok = true;
      for (int j = 0; ok && j < n; ++j) {
        const int s = j % C::kVStages;
        const uint32_t vbase = base + C::kVOff + s * C::kTileBytes;
        for (int t = 0; ok && t < ntile; ++t) {
          // QK_t(j+1) is on the softmax's critical path and this P·V is not (its P buffer is
          // reused only a block later): let that QK reach the tensor core first (bounded;
          // the order never affects results)
          if (j + 1 < n) {
            for (int spin = 0; spin < 4096 && qk_issued[t] < j + 2 && !*abort_flag; ++spin) __nanosleep(32);
          }
          if (!mbar_wait(bar(C::kBarPFull + t), static_cast<uint32_t>(j) & 1, abort_flag) ||
              (t == 0 && !mbar_wait(bar(C::kBarVFull + s), static_cast<uint32_t>(j / C::kVStages) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pcol = tmem + C::kColP + 64 * t;
          const uint32_t ocol = tmem + (t ? C::kColO1 : C::kColO0);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // B = V tile, MN-major: 16 key rows per step (2048 B), D-halves one swizzle column apart
            mma_f16_ts(ocol, pcol + kk * 8, sdesc_sw128(vbase + kk * 2048, C::kSubBytes, 1024), idesc_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(C::kBarPVDone + t));
          if (t == ntile - 1) mma_commit(bar(C::kBarVEmpty + s));  // both tiles' P·Vs of V_j retired
          if (j == n - 1) mma_commit(bar(C::kBarOFinal + t));
        }
      }
      mma_commit(bar(C::kBarDrain + 1));
      mbar_wait_drain(bar(C::kBarDrain + 1), 0);
    }
  } else if (warp < 8) {
    // ---------------------------------------------------------------- softmax warps
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool tile_live = t < ntile;
    const int nt = tile_live ? n : 0;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t i_glob = (int64_t)(2 * pr + t) * kTile + row;
    const float kNegInf = -__int_as_float(0x7f800000);
    const float c = p.scale * 1.4426950408889634f;  // score -> log2 domain
    const uint32_t s_col = tmem + lane_off + C::kColS;
    const uint32_t o_col = tmem + lane_off + (t ? C::kColO1 : C::kColO0);
    const uint32_t p_col = tmem + lane_off + C::kColP + 64 * t;
    const int valid_last = p.Skv - (n - 1) * kTile;  // key columns of the last tile inside S_kv

    float m_ref = kNegInf, m_true = kNegInf, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < nt; ++j) {
      ok = warp_wait(bar(C::kBarSFull + t), static_cast<uint32_t>(j) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      float sv[128];
      {
        uint32_t rr[128];
        tmem_ld128_wait(s_col, rr);
#pragma unroll
        for (int x = 0; x < 128; ++x) sv[x] = __uint_as_float(rr[x]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarSFree + t));

      if (j == n - 1 && valid_last < kTile) {  // tail tile: keys past S_kv take no part
#pragma unroll
        for (int x = 0; x < 128; ++x)
          if (x >= valid_last) sv[x] = kNegInf;
      }
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = sv[i];
#pragma unroll
      for (int x = 8; x < 128; x += 16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = fmax3(a[i], sv[x + i], sv[x + 8 + i]);
      }
      const float rmax = fmaxf(fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3])), fmaxf(fmaxf(a[4], a[5]), fmaxf(a[6], a[7])));

      const float m_new = fmaxf(m_true, rmax);
      const bool upd = (m_new > m_ref) && (m_ref == kNegInf || (m_new - m_ref) * c > 8.0f);
      const float alpha = upd ? ex2((m_ref - m_new) * c) : 1.0f;
      const bool need = upd && (j > 0) && (m_ref != kNegInf);
      if (upd) {
        l *= alpha;
        m_ref = m_new;
      }
      m_true = m_new;
      const float mc = (m_ref == kNegInf) ? 0.f : m_ref * c;
      const uint64_t cc = pack_f32x2(c, c);
      const uint64_t nm = pack_f32x2(-mc, -mc);
      uint32_t pk[64];
      uint64_t acc[2] = {0ull, 0ull};  // packed partial row sums: two pairs of lanes
#pragma unroll
      for (int x = 0; x < 64; ++x) {
        float z0, z1;
        fma_f32x2(sv[2 * x], sv[2 * x + 1], cc, nm, z0, z1);
        const float p0 = ex2(z0);
        const float p1 = ex2(z1);
        add_f32x2(acc[x & 1], p0, p1);
        pk[x] = pack_bf16x2(p0, p1);
      }
      l += sum_f32x2(acc[0]) + sum_f32x2(acc[1]);

      // P_t and O_t are free once the previous block's P·V has retired
      if (j > 0) {
        ok = warp_wait(bar(C::kBarPVDone + t), static_cast<uint32_t>(j - 1) & 1, abort_flag);
        if (!ok) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
          uint32_t rr[32];
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            tmem_ld32_wait(o_col + ch * 32, rr);
#pragma unroll
            for (int x = 0; x < 32; ++x) rr[x] = __float_as_uint(__uint_as_float(rr[x]) * alpha);
            tmem_st32(o_col + ch * 32, rr);
          }
        }
      }
      tmem_st64(p_col, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarPFull + t));
    }

    // ------------------------------------------------------------ epilogue
    bool have_o = ok && nt > 0;
    if (have_o) {
      // a dedicated single-use barrier: pv_done's parity cannot tell PV(n-1) from PV(n-3)
      have_o = warp_wait(bar(C::kBarOFinal + t), 0, abort_flag);
      tc_fence_after();
    }
    const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
    // O -> bf16 staged in this tile's Q buffer (its last QK has retired) in the
    // 128-byte-swizzled layout of the output tensor map, then written by two TMA stores
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint32_t stage = base + C::kQOff + t * C::kTileBytes + hf * C::kSubBytes;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t rr[32];
        if (have_o) {
          tmem_ld32_wait(o_col + hf * 64 + ch * 32, rr);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) rr[x] = 0u;
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          float f[8];
#pragma unroll
          for (int y = 0; y < 8; ++y) f[y] = __uint_as_float(rr[8 * x + y]) * inv_l;
          const int chunk = ch * 4 + x;  // 16-byte chunk of this row's 128-byte line
          const uint32_t dst = stage + row * 128 + ((chunk ^ (row & 7)) << 4);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(dst), "r"(pack_bf16x2(f[0], f[1])),
                       "r"(pack_bf16x2(f[2], f[3])), "r"(pack_bf16x2(f[4], f[5])), "r"(pack_bf16x2(f[6], f[7]))
                       : "memory");
        }
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + t, 128);
    if (quarter == 0 && lane == 0) {
      if (tile_live) {
        tma_store_4d(&p.tm_o, base + C::kQOff + t * C::kTileBytes, 0, (2 * pr + t) * kTile, h, b);
        tma_store_4d(&p.tm_o, base + C::kQOff + t * C::kTileBytes + C::kSubBytes, 64, (2 * pr + t) * kTile, h, b);
        bulk_commit_group();
      }
      bulk_wait_read_all();  // shared memory must outlive the stores' reads
    }
    if (tile_live && i_glob < p.Sq && (p.softmax_max || p.softmax_sum)) {
      const int64_t sidx = ((int64_t)b * p.Nq + h) * p.Sq + i_glob;
      const bool live = (m_true != kNegInf) && (l > 0.f);
      if (p.softmax_max) p.softmax_max[sidx] = live ? m_true * p.scale : kNegInf;
      if (p.softmax_sum) p.softmax_sum[sidx] = live ? l * ex2((m_ref - m_true) * c) : 0.f;  // against the true max
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kWarpQK) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace qbsa
