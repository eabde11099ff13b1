// Dense bf16 fused attention forward for sm_100a, two query tiles per CTA, under masks.
//
// Computes Softmax(Mask(Q·Kᵀ·scale))·V (npu_fusion_attention guide, "昇腾 NPU 融合注意力算子详解与
// 迁移指南", §2 算子数学原理) for D = 128 without an explicit atten_mask or pse, in the BNSD,
// BSND and TND layouts (§4.1) under sparse_mode 0 (band of pre_tokens / next_tokens), 2 and
// 3 (causal, §4.3), per sequence for TND, with the outputs of §5 (attention_out,
// softmax_max, softmax_sum).  The unmasked case runs on attn_pair_kernel (attn_pair.cuh),
// whose layout and warp roles this kernel shares; attn_dense_kernel serves atten_mask, pse,
// D = 64 and block masks.
//
// One CTA owns two adjacent 128-row query tiles of one (batch or sequence, head).  Each
// tile visits its own K-tile range (the schedule of schedule.cuh: causal and band tiles
// outside the range are skipped, tiles partly inside it get an element mask); the CTA
// walks the union of the two ranges, so every K/V tile is loaded once for the tiles that
// need it, and the two tiles take turns on one TMEM score buffer.
//
// CTA = 12 warps, the roles of attn_pair_kernel plus an idle warp that completes the third
// warpgroup: after set-up that warpgroup gives registers back (setmaxnreg, 168 -> 64 per
// thread) and the two softmax warpgroups take them (168 -> 216), which removes the softmax
// loop's spills (this kernel's per-row mask state needs more registers than the unmasked one):
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1 (row 32*(warp%4)+lane, lazy O rescale);
//                    epilogue: O / l staged in the tile's Q buffer and written by TMA stores
//                    (BNSD / BSND), or stored row by row (TND, whose tiles may end inside the
//                    next sequence's rows).
//   warp 8           TMA producer: the Q tiles once, then the union's K and V tiles.
//   warp 9           TMEM owner + QK issuer, for each tile whose range holds key tile j.
//   warp 10          P·V issuer, each P·V queued behind the same tile's next QK.
//   warp 11          no work after set-up.
// TMEM columns: O0 [0,128) O1 [128,256) S [256,384) P0 [384,448) P1 [448,512).
//
// CTA order: query heads in groups whose K/V fit in about 48 MB of L2; inside a group the
// heaviest pairs first (the last pairs of a causal sequence, the longest sequences), heads
// fastest.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "attn_dense.cuh"
#include "attn_pair.cuh"
#include "ptx_sm100.cuh"
#include "schedule.cuh"

namespace qbsa {

struct PairMaskedParams {
  CUtensorMap tm_q;  // 4-D {128, rows, heads, batch}, box {64, 128, 1, 1}, bf16, SW128
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  CUtensorMap tm_o;  // the output, same layout and box as tm_q (BNSD / BSND)
  __nv_bfloat16* out;  // TND: rows stored directly
  float* softmax_max;  // [B, Nq, Sq] ([Nq, T] for TND) or nullptr
  float* softmax_sum;
  int64_t o_row_stride, o_head_stride;           // TND output strides (elements)
  int64_t stat_head_stride, stat_batch_stride;   // statistics strides (elements)
  int64_t pre_tokens, next_tokens;
  int B, Nq, Nkv, Sq, Skv, group;
  int sparse_mode;
  int tnd;       // 1: varlen TND
  int n_qtiles;  // BNSD / BSND: ceil(Sq / 128)
  int n_pair;    // BNSD / BSND: ceil(n_qtiles / 2)
  int n_rank;    // query-tile pairs per head (all batches / sequences)
  int head_grp;  // query heads per L2 group
  float scale;
  // TND tables (sequences in processing order)
  int n_seq;
  int seq_q_start[kMaxSeqs];
  int seq_q_len[kMaxSeqs];
  int seq_kv_start[kMaxSeqs];
  int seq_kv_len[kMaxSeqs];
  int seq_pair_start[kMaxSeqs + 1];
};

struct PairWork {
  int b, h, pr;
  int ntiles;       // query tiles of the (batch or sequence, head)
  int64_t q_row0;   // tensor-map row coordinate of query row 0 of the sequence
  int64_t kv_row0;  // tensor-map row coordinate of key row 0 of the sequence
  int coord_b;      // tensor-map batch coordinate
  int64_t sq, skv;  // sequence lengths
  int64_t tok0;     // TND: first token of the sequence (output / statistics rows)
};

__device__ __forceinline__ PairWork pair_work(const PairMaskedParams& p) {
  PairWork w;
  // head groups (L2 reuse of K/V), heaviest pairs first, heads fastest inside a group
  const int64_t per_group = (int64_t)p.head_grp * p.n_rank;
  const int grp = static_cast<int>(blockIdx.x / per_group);
  const int h0 = grp * p.head_grp;
  const int hcount = min(p.head_grp, p.Nq - h0);
  const int off = static_cast<int>(blockIdx.x - grp * per_group);
  const int r = off / hcount;
  w.h = h0 + off % hcount;
  if (!p.tnd) {
    w.b = r % p.B;
    w.pr = p.n_pair - 1 - r / p.B;
    w.ntiles = p.n_qtiles;
    w.q_row0 = 0;
    w.kv_row0 = 0;
    w.coord_b = w.b;
    w.sq = p.Sq;
    w.skv = p.Skv;
    w.tok0 = 0;
  } else {
    int lo = 0, hi = p.n_seq - 1;
    while (lo < hi) {  // last i with seq_pair_start[i] <= r
      const int mid = (lo + hi + 1) >> 1;
      if (p.seq_pair_start[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int npair = p.seq_pair_start[lo + 1] - p.seq_pair_start[lo];
    w.b = 0;
    w.pr = npair - 1 - (r - p.seq_pair_start[lo]);
    w.q_row0 = p.seq_q_start[lo];
    w.kv_row0 = p.seq_kv_start[lo];
    w.coord_b = 0;
    w.sq = p.seq_q_len[lo];
    w.skv = p.seq_kv_len[lo];
    w.ntiles = static_cast<int>((w.sq + kTile - 1) / kTile);
    w.tok0 = p.seq_q_start[lo];
  }
  return w;
}

struct PairMaskedCfg {
  static constexpr int kThreads = 384;
  static constexpr int kRegSoftmax = 216, kRegHelper = 64;  // per thread, after set-up
};
static_assert(2 * 128 * PairMaskedCfg::kRegSoftmax + 128 * PairMaskedCfg::kRegHelper <= PairMaskedCfg::kThreads * 168,
              "register shares above what a 168-register launch holds");

__global__ void __launch_bounds__(384, 1) attn_pair_masked_kernel(const __grid_constant__ PairMaskedParams p) {
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

  const PairWork w = pair_work(p);
  const int h = w.h, g = h / p.group;
  const Band band = band_of(p.sparse_mode, p.pre_tokens, p.next_tokens, w.sq, w.skv);
  // per tile: live (exists) and its K-tile range [kb, ke)
  const bool live0 = 2 * w.pr < w.ntiles, live1 = 2 * w.pr + 1 < w.ntiles;
  const TileRange tr0 = live0 ? tile_range(2 * w.pr, w.sq, w.skv, band) : TileRange{0, 0, 0, 0};
  const TileRange tr1 = live1 ? tile_range(2 * w.pr + 1, w.sq, w.skv, band) : TileRange{0, 0, 0, 0};
  const int kb0 = tr0.kt_begin, ke0 = tr0.kt_end, kb1 = tr1.kt_begin, ke1 = tr1.kt_end;
  const int n0 = ke0 - kb0, n1 = ke1 - kb1;
  // the union of the two (overlapping or adjacent) ranges, walked by producer and issuers
  const int ub = (n0 > 0 && n1 > 0) ? min(kb0, kb1) : (n0 > 0 ? kb0 : kb1);
  const int ue = (n0 > 0 && n1 > 0) ? max(ke0, ke1) : (n0 > 0 ? ke0 : ke1);
  const int nj = (n0 > 0 || n1 > 0) ? ue - ub : 0;

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
      if (!p.tnd) tma_prefetch_desc(&p.tm_o);
    }
  } else if (warp == C::kWarpQK) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 8) {
    regs_dec<PairMaskedCfg::kRegHelper>();
    if (warp == C::kWarpProducer) {
      // ---------------------------------------------------------------- producer
      if (lane == 0 && nj > 0) {
        const uint64_t pol_q = l2_policy_evict_first();
        const uint64_t pol_kv = l2_policy_evict_last();
        mbar_arrive_expect_tx(bar(C::kBarQFull), C::kTileBytes * ((n0 > 0) + (n1 > 0)));
        for (int t = 0; t < 2; ++t) {
          if ((t ? n1 : n0) == 0) continue;
          const int qrow = static_cast<int>(w.q_row0 + (int64_t)(2 * w.pr + t) * kTile);
          for (int sub = 0; sub < 2; ++sub)
            tma_load_4d(base + C::kQOff + t * C::kTileBytes + sub * C::kSubBytes, &p.tm_q, bar(C::kBarQFull),
                        sub * 64, qrow, h, w.coord_b, pol_q);
        }
        int kq = 0, vq = 0;  // K / V copies issued
        for (int jj = 0; jj < nj; ++jj) {
          const int kv_row = static_cast<int>(w.kv_row0 + (int64_t)(ub + jj) * kTile);
          const int sk = jj % C::kKStages, sv = jj % C::kVStages;
          if (jj >= C::kKStages &&
              !mbar_wait(bar(C::kBarKEmpty + sk), (static_cast<uint32_t>(jj / C::kKStages) & 1) ^ 1, abort_flag))
            break;
          mbar_arrive_expect_tx(bar(C::kBarKFull + sk), C::kTileBytes);
          for (int sub = 0; sub < 2; ++sub)
            tma_load_4d(base + C::kKOff + sk * C::kTileBytes + sub * C::kSubBytes, &p.tm_k, bar(C::kBarKFull + sk),
                        sub * 64, kv_row, g, w.coord_b, pol_kv);
          ++kq;
          if (jj >= C::kVStages &&
              !mbar_wait(bar(C::kBarVEmpty + sv), (static_cast<uint32_t>(jj / C::kVStages) & 1) ^ 1, abort_flag))
            break;
          mbar_arrive_expect_tx(bar(C::kBarVFull + sv), C::kTileBytes);
          for (int sub = 0; sub < 2; ++sub)
            tma_load_4d(base + C::kVOff + sv * C::kTileBytes + sub * C::kSubBytes, &p.tm_v, bar(C::kBarVFull + sv),
                        sub * 64, kv_row, g, w.coord_b, pol_kv);
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
      if (lane == 0 && nj > 0) {
        constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false);
        bool ok = mbar_wait(bar(C::kBarQFull), 0, abort_flag);
        int prev_t = -1, prev_l = 0;  // reader of the S buffer's current contents (tile, local block)
        for (int jj = 0; ok && jj < nj; ++jj) {
          const int j = ub + jj;
          const int s = jj % C::kKStages;
          if (!mbar_wait(bar(C::kBarKFull + s), static_cast<uint32_t>(jj / C::kKStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t kbase = base + C::kKOff + s * C::kTileBytes;
  #pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int kb = t ? kb1 : kb0, ke = t ? ke1 : ke0;
            if (!ok || j < kb || j >= ke) continue;
            const int lt = j - kb;
            if (prev_t >= 0 && !mbar_wait(bar(C::kBarSFree + prev_t), static_cast<uint32_t>(prev_l) & 1, abort_flag)) {
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
            qk_issued[t] = lt + 1;  // lets the PV issuer queue behind this QK
            prev_t = t;
            prev_l = lt;
          }
          if (!ok) break;
          mma_commit(bar(C::kBarKEmpty + s));  // every QK of K_j retired
        }
        // every MMA issued above has retired before TMEM can be released
        mma_commit(bar(C::kBarDrain));
        mbar_wait_drain(bar(C::kBarDrain), 0);
      }
    } else if (warp == C::kWarpPV) {
      // ---------------------------------------------------------------- PV issuer
      if (lane == 0 && nj > 0) {
        constexpr uint32_t idesc_pv = idesc_bf16(128, 128, true);
        bool ok = true;
        for (int jj = 0; ok && jj < nj; ++jj) {
          const int j = ub + jj;
          const int s = jj % C::kVStages;
          const uint32_t vbase = base + C::kVOff + s * C::kTileBytes;
          bool v_ready = false;
  #pragma unroll
          for (int t = 0; t < 2; ++t) {
            const int kb = t ? kb1 : kb0, ke = t ? ke1 : ke0;
            if (!ok || j < kb || j >= ke) continue;
            const int lt = j - kb;
            const int nt = ke - kb;
            // QK_t(lt+1) is on the softmax's critical path and this P·V is not (its P buffer is
            // reused only a block later): let that QK reach the tensor core first (bounded;
            // the order never affects results)
            if (lt + 1 < nt) {
              for (int spin = 0; spin < 4096 && qk_issued[t] < lt + 2 && !*abort_flag; ++spin) __nanosleep(32);
            }
            if (!mbar_wait(bar(C::kBarPFull + t), static_cast<uint32_t>(lt) & 1, abort_flag) ||
                (!v_ready &&
                 !mbar_wait(bar(C::kBarVFull + s), static_cast<uint32_t>(jj / C::kVStages) & 1, abort_flag))) {
              ok = false;
              break;
            }
            v_ready = true;
            tc_fence_after();
            const uint32_t pcol = tmem + C::kColP + 64 * t;
            const uint32_t ocol = tmem + (t ? C::kColO1 : C::kColO0);
  #pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              // B = V tile, MN-major: 16 key rows per step (2048 B), D-halves one swizzle column apart
              mma_f16_ts(ocol, pcol + kk * 8, sdesc_sw128(vbase + kk * 2048, C::kSubBytes, 1024), idesc_pv,
                         (lt > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(bar(C::kBarPVDone + t));
            if (lt == nt - 1) mma_commit(bar(C::kBarOFinal + t));
          }
          // (the two ranges overlap or abut, so some tile needs every key tile of the union;
          // should none, the copy must still land before its stage is handed back)
          if (ok && !v_ready)
            ok = mbar_wait(bar(C::kBarVFull + s), static_cast<uint32_t>(jj / C::kVStages) & 1, abort_flag);
          if (!ok) break;
          mma_commit(bar(C::kBarVEmpty + s));  // every P·V of V_j retired
        }
        mma_commit(bar(C::kBarDrain + 1));
        mbar_wait_drain(bar(C::kBarDrain + 1), 0);
      }
    }
  } else {
    regs_inc<PairMaskedCfg::kRegSoftmax>();
    // ---------------------------------------------------------------- softmax warps
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const bool tile_live = t ? live1 : live0;
    const TileRange my = t ? tr1 : tr0;
    const int nt = my.kt_end - my.kt_begin;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int i_loc = (2 * w.pr + t) * kTile + row;  // query index inside the sequence (< 2^31)
    const float kNegInf = -__int_as_float(0x7f800000);
    const float c = p.scale * 1.4426950408889634f;  // score -> log2 domain
    const uint32_t s_col = tmem + lane_off + C::kColS;
    const uint32_t o_col = tmem + lane_off + (t ? C::kColO1 : C::kColO0);
    const uint32_t p_col = tmem + lane_off + C::kColP + 64 * t;
    // this row's keys [j_lo, j_hi] of the sequence (band or causal, and below S_kv), clamped
    // to [-1, S_kv] so they fit in 32 bits
    const int j_lo = static_cast<int>(max64(-1, min64(w.skv, (int64_t)i_loc - band.lo_off)));
    const int j_hi = static_cast<int>(max64(-1, min64(w.skv - 1, (int64_t)i_loc + band.hi_off)));

    float m_ref = kNegInf, m_true = kNegInf, l = 0.f;
    bool ok = true;
    for (int lt = 0; ok && lt < nt; ++lt) {
      const int kt = my.kt_begin + lt;
      ok = warp_wait(bar(C::kBarSFull + t), static_cast<uint32_t>(lt) & 1, abort_flag);
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

      if (kt < my.full_begin || kt >= my.full_end) {
        // a tile partly outside the mask (band / causal edge, or past S_kv): element mask
        const int col0 = kt * kTile;
        const int clo = j_lo - col0, chi = j_hi - col0;
#pragma unroll
        for (int x = 0; x < 128; ++x)
          if (x < clo || x > chi) sv[x] = kNegInf;
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
      const bool need = upd && (lt > 0) && (m_ref != kNegInf);
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
      if (lt > 0) {
        ok = warp_wait(bar(C::kBarPVDone + t), static_cast<uint32_t>(lt - 1) & 1, abort_flag);
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
    const PairWork we = pair_work(p);  // recomputed rather than held in registers through the loop
    const bool row_valid = tile_live && i_loc < we.sq;
    if (p.tnd) {
      // rows past the sequence's end belong to the next sequence: store row by row
      __nv_bfloat16* orow =
          row_valid ? p.out + (we.tok0 + i_loc) * p.o_row_stride + (int64_t)we.h * p.o_head_stride : nullptr;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rr[32];
        if (have_o) {
          tmem_ld32_wait(o_col + ch * 32, rr);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) rr[x] = 0u;
        }
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            float f[8];
#pragma unroll
            for (int y = 0; y < 8; ++y) f[y] = __uint_as_float(rr[8 * x + y]) * inv_l;
            dst[x] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                pack_bf16x2(f[6], f[7]));
          }
        }
      }
    } else {
      // O -> bf16 staged in this tile's Q buffer (its last QK has retired, and it was never
      // loaded if the tile visits no key tile) in the 128-byte-swizzled layout of the output
      // tensor map, then written by two TMA stores (rows past S_q are clipped)
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
        if (tile_live && (ok || nt == 0)) {
          const int qrow = (2 * we.pr + t) * kTile;
          tma_store_4d(&p.tm_o, base + C::kQOff + t * C::kTileBytes, 0, qrow, we.h, we.coord_b);
          tma_store_4d(&p.tm_o, base + C::kQOff + t * C::kTileBytes + C::kSubBytes, 64, qrow, we.h, we.coord_b);
          bulk_commit_group();
        }
        bulk_wait_read_all();  // shared memory must outlive the stores' reads
      }
    }
    if (row_valid && (p.softmax_max || p.softmax_sum)) {
      const int64_t sidx = (int64_t)we.b * p.stat_batch_stride + (int64_t)we.h * p.stat_head_stride + we.tok0 + i_loc;
      const bool rlive = (m_true != kNegInf) && (l > 0.f);
      if (p.softmax_max) p.softmax_max[sidx] = rlive ? m_true * p.scale : kNegInf;
      if (p.softmax_sum) p.softmax_sum[sidx] = rlive ? l * ex2((m_ref - m_true) * c) : 0.f;  // against the true max
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
