// Quantized block-sparse attention forward (EagleQBSA) for sm_100a.
//
// EagleQBSA article ("昇腾MindIE SD高性能量化稀疏联合注意力EagleQBSA,视频生成端到端加速1.6倍"):
// Q and K arrive as INT8 with one scale per 128-token block, V as FP8 E4M3 with one
// scale per channel, and P is rounded to FP8 before P·V (section
// "EagleQBSA量化叠加稀疏方案设计", Fig 2.1); only the 128x128 blocks selected by the
// block-sparse mask are computed (section "背景介绍"; block_sparse_mask and
// block_shape=[128,128] in section "MindIE SD调用方式").
//
// One CTA per (batch, head, pair of 128-row query blocks).  The two query tiles share
// the tensor core and take turns on the special-function unit: while one tile's
// warps load scores and reduce row maxima, the other tile's warps are in their
// exponentials.  Each tile's row of the block mask is first compacted into the
// ascending list of kept key blocks in shared memory.  Then:
//   warps 0..3  softmax of tile 0, warps 4..7 softmax of tile 1: one thread per query
//               row (TMEM lane 32*(warp%4)+lane), all 128 key columns of a block.
//               Exact s32 -> f32 (|dot| < 2^24), dequantisation constant
//               c = s_q * s_k * scale * log2(e) (s_k fetched a block ahead), online
//               softmax whose weights p = 2^(z - R) use a power-of-two reference R
//               re-set to ceil(running max) only when the max exceeds it by more than 8
//               (exact power-of-two rescales of O and L, rare);
//               P -> FP16 -> E4M3 into TMEM.  A last kept block that runs past S_kv
//               (ragged S_kv) is handled by an out-of-line copy of the step that masks
//               the keys beyond S_kv, so the main loop carries no masking code.
//               Epilogue O * v_scale / L -> bf16 staged
//               in the tile's Q buffer (free by then) and a second buffer, written by
//               TMA stores.
//   warp 8      TMA producer: Q of both tiles once; K and V tiles of the kept blocks
//               of both tiles, interleaved (t0 j, t1 j, t0 j+1, ...), into a 4-stage K
//               ring (a stage is free once its QK retired) and a 5-stage V ring (free
//               once its P·V retired), so K is fetched about two blocks ahead.
//   warp 9      TMEM owner + QK issuer: S = Q8_t K8ᵀ (kind::i8, s32 into the one
//               shared S buffer) once the S buffer's previous reader is done.
//   warp 10     PV issuer: [O_t | L_t] += P8_t [V8 | 1] as one N = 144 MMA
//               (kind::f8f6f4, A = P8 from TMEM, B MN-major: V8's 128 channels plus a
//               16-column ones block in shared memory), so L is exactly Σ p8.
// The two issuers block independently while the tensor core drains their queues.
// TMEM columns: O0|L0 [0,144) S [160,288) O1|L1 [288,432) P0 [448,480) P1 [480,512).
//
// CTA order: query heads in groups whose K8/V8 fit in about 48 MB of L2, query-block
// pairs in order, heads fastest inside a group.
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
  CUtensorMap tm_o;  // bf16 output {128, Sq, Nq, B}, box {64, 128, 1, 1}, SW128
  const float* q_scale;   // [B, Nq, nqb]
  const float* k_scale;   // [B, Nkv, nkb]
  const float* v_scale;   // [B, Nkv, 128]
  const uint8_t* block_mask;  // [B, Nq, nqb, nkb], 1 = compute
  __nv_bfloat16* out;     // [B, Nq, Sq, 128]
  float* softmax_max;     // [B, Nq, Sq] or nullptr
  float* softmax_sum;
  int B, Nq, Nkv, Sq, Skv, group, nqb, nkb;
  int n_pair;             // ceil(nqb / 2) query-block pairs per (batch, head)
  int n_rank;             // B * n_pair
  int head_grp;           // query heads per L2 group
  int mask_v16;           // mask rows are 16-byte aligned with nkb % 16 == 0 (vector compaction)
  float scale_log2;       // scale * log2(e)
};

struct QbsaCfg {
  static constexpr int D = 128;
  static constexpr int kKStages = 4;                // K tiles in flight
  static constexpr int kVStages = 5;                // V tiles in flight
  static constexpr int kTileBytes = kTile * 128;    // 128 rows x 128 bytes
  static constexpr int kQOff = 0;                   // Q of tile 0, then tile 1
  static constexpr int kKOff = kQOff + 2 * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kEOff = kVOff + kVStages * kTileBytes;     // [2] epilogue staging, columns 64..127
  static constexpr int kOnesOff = kEOff + 2 * kTileBytes;           // 32 rows x 128 B of E4M3 1.0
  static constexpr int kListOff = kOnesOff + 4096;                 // uint16 [2][kMax] kept blocks
  static constexpr int kVscOff = kListOff + 2 * kQbsaMaxKBlocks * 2;  // float [128] value scales
  static constexpr int kBarOff = kVscOff + 128 * 4;
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
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;  // tmem addr, abort flag, counts[2]
  static constexpr int kSmemBytes = kMiscOff + 32 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // O_t|L_t at kColO[t] (L_t = its column 128), P_t at kColP + 32 t
  static constexpr uint32_t kColO0 = 0, kColS = 160, kColO1 = 288, kColP = 448;
  static constexpr int kThreads = 352;
  static constexpr int kWarpProducer = 8, kWarpQK = 9, kWarpPV = 10;
};
static_assert(QbsaCfg::kSmemBytes <= 232448, "shared memory above the 227 KB opt-in limit");
// TMA tiles and UMMA operands use the 128-byte swizzle, whose pattern repeats every 1024 bytes
static_assert(QbsaCfg::kKOff % 1024 == 0 && QbsaCfg::kVOff % 1024 == 0 && QbsaCfg::kEOff % 1024 == 0 &&
                  QbsaCfg::kOnesOff % 1024 == 0 && QbsaCfg::kTileBytes % 1024 == 0,
              "swizzled buffers must start on 1024-byte boundaries");

// Compact one row of the block mask (n_kb bytes, nonzero = keep) into ascending indices.
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

// Same result for a 16-byte aligned row with n_kb % 16 == 0 and n_kb <= 2048: every lane
// loads its 16-byte chunks at once (one memory round trip), counts the nonzero bytes,
// and a warp prefix sum places each lane's indices.
__device__ __forceinline__ int compact_mask_row_v16(const uint8_t* row, int n_kb, uint16_t* list, int lane) {
  const int n_chunks = n_kb >> 4;
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  uint4 v[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = lane + 32 * i;
    v[i] = (c < n_chunks) ? __ldg(r4 + c) : make_uint4(0u, 0u, 0u, 0u);
  }
  int count = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (32 * i >= n_chunks) break;
    const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
    uint32_t nz[4];
    int mine = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      nz[k] = (((w[k] & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | w[k]) & 0x80808080u;  // bit 7 of a byte: byte != 0
      mine += __popc(nz[k]);
    }
    int incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += y;
    }
    int pos = count + incl - mine;
    const int j0 = (lane + 32 * i) * 16;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      for (uint32_t m = nz[k]; m != 0u; m &= m - 1u)
        list[pos++] = static_cast<uint16_t>(j0 + 4 * k + ((__ffs(m) - 1) >> 3));
    }
    count += __shfl_sync(0xffffffffu, incl, 31);
  }
  return count;
}

struct QbsaTailResult {
  float m, ref;
  int ok;
};

// The softmax step of a row's last kept block when that block runs past S_kv (only the last
// can: the kept lists are ascending).  Out of line so that the main loop carries no code for
// the masking; called by the whole warp, at most once per row.  Same arithmetic as the loop.
__device__ __noinline__ QbsaTailResult qbsa_tail_block(uint32_t s_col, uint32_t o_col, uint32_t p_col,
                                                       uint32_t bar_sfull, uint32_t bar_sfree, uint32_t bar_pvdone,
                                                       uint32_t bar_pfull, int j, float cst, int valid, float m,
                                                       float ref, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  const float kNegInf = -__int_as_float(0x7f800000);
  QbsaTailResult r{m, ref, 0};
  if (!warp_wait(bar_sfull, static_cast<uint32_t>(j) & 1, abort_flag)) return r;
  tc_fence_after();
  uint32_t sv[128];
  tmem_ld128_wait(s_col, sv);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar_sfree);
  const bool pos = cst >= 0.f;
  const uint32_t pad = pos ? 0x80000000u : 0x7fffffffu;  // keys past S_kv take no part in the max
#pragma unroll
  for (int x = 0; x < 128; ++x)
    if (x >= valid) sv[x] = pad;
  const float m_blk = __int2float_rn(pos ? imax128(sv) : imin128(sv)) * cst;
  m = fmaxf(m, m_blk);
  const bool upd = (ref == kNegInf) || (m > ref + 8.0f);
  const float new_ref = upd ? ceilf(m) : ref;
  const bool need = upd && (ref != kNegInf);
  const int dexp = need ? static_cast<int>(ref - new_ref) : 0;
  const float a = (dexp < -126) ? 0.f : __int_as_float((127 + dexp) << 23);
  ref = new_ref;
  const uint64_t cc = pack_f32x2(cst, cst);
  const uint64_t nr = pack_f32x2(-ref, -ref);
  uint32_t pk[32];
#pragma unroll
  for (int x = 0; x < 32; ++x) {
    pk[x] = i2f_fma_exp2_e4m3x4(sv[4 * x], sv[4 * x + 1], sv[4 * x + 2], sv[4 * x + 3], cc, nr);
    const int keep = min(max(valid - 4 * x, 0), 4);  // zero the weights of keys past S_kv
    pk[x] &= (keep == 4) ? 0xffffffffu : ((1u << (8 * keep)) - 1u);
  }
  if (j > 0) {
    if (!warp_wait(bar_pvdone, static_cast<uint32_t>(j - 1) & 1, abort_flag)) return r;
    tc_fence_after();
    if (__any_sync(0xffffffffu, need)) {
      uint32_t rr[32];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        tmem_ld32_wait(o_col + ch * 32, rr);
#pragma unroll
        for (int x = 0; x < 32; ++x) rr[x] = __float_as_uint(__uint_as_float(rr[x]) * a);
        tmem_st32(o_col + ch * 32, rr);
      }
      tmem_st1(o_col + 128, __float_as_uint(__uint_as_float(tmem_ld1_wait(o_col + 128)) * a));
    }
  }
  tmem_st32(p_col, pk);
  tmem_st_wait();
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(bar_pfull);
  r.m = m;
  r.ref = ref;
  r.ok = 1;
  return r;
}

__global__ void __launch_bounds__(352, 1) attn_qbsa_kernel(const __grid_constant__ QbsaParams p) {
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
  int* count_slot = reinterpret_cast<int*>(smem + C::kMiscOff + 8);  // [2]
  volatile int* qk_issued = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 16);  // [2] QKs issued per tile
  uint16_t* lists = reinterpret_cast<uint16_t*>(smem + C::kListOff);
  float* vsc = reinterpret_cast<float*>(smem + C::kVscOff);

  // head groups (L2 reuse of K/V), query-block pairs in order, heads fastest in a group
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

  if (warp == 0 || warp == 4) {
    // kept-block list of tile t
    const int t = warp >> 2;
    const int qb = 2 * pr + t;
    uint16_t* list = lists + t * kQbsaMaxKBlocks;
    int cnt = 0;
    if (qb < p.nqb) {
      const uint8_t* mrow = p.block_mask + (((int64_t)b * p.Nq + h) * p.nqb + qb) * p.nkb;
      cnt = p.mask_v16 ? compact_mask_row_v16(mrow, p.nkb, list, lane) : compact_mask_row(mrow, p.nkb, list, lane);
    }
    if (lane == 0) count_slot[t] = cnt;
  } else if (warp == 1) {
    // the ones block (E4M3 1.0 = 0x38) that turns the P·V MMA's columns 128..143 into Σ p8
    uint32_t* ones = reinterpret_cast<uint32_t*>(smem + C::kOnesOff);
    for (int i = lane; i < 1024; i += 32) ones[i] = 0x38383838u;
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  } else if (warp == 2) {
    const float* vs = p.v_scale + ((int64_t)b * p.Nkv + g) * 128;
    for (int i = lane; i < 128; i += 32) vsc[i] = vs[i];
  } else if (warp == C::kWarpProducer) {
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
      }
      mbar_init(bar(C::kBarDrain), 1);
      mbar_init(bar(C::kBarDrain + 1), 1);
      fence_mbar_init();
      tma_prefetch_desc(&p.tm_q);
      tma_prefetch_desc(&p.tm_k);
      tma_prefetch_desc(&p.tm_v);
    }
  } else if (warp == C::kWarpQK) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n0 = count_slot[0], n1 = count_slot[1];
  const int n_max = max(n0, n1);

  if (warp == C::kWarpProducer) {
    // ---------------------------------------------------------------- producer
    if (lane == 0 && n_max > 0) {
      const uint64_t pol_q = l2_policy_evict_first();
      const uint64_t pol_kv = l2_policy_evict_last();
      mbar_arrive_expect_tx(bar(C::kBarQFull), C::kTileBytes * ((n0 > 0) + (n1 > 0)));
      if (n0 > 0) tma_load_4d(base + C::kQOff, &p.tm_q, bar(C::kBarQFull), 0, (2 * pr) * kTile, h, b, pol_q);
      if (n1 > 0)
        tma_load_4d(base + C::kQOff + C::kTileBytes, &p.tm_q, bar(C::kBarQFull), 0, (2 * pr + 1) * kTile, h, b,
                    pol_q);
      int seq = 0;
      bool ok = true;
      for (int j = 0; ok && j < n_max; ++j) {
        for (int t = 0; t < 2; ++t) {
          if (j >= (t ? n1 : n0)) continue;
          const int kv_row = static_cast<int>(lists[t * kQbsaMaxKBlocks + j]) * kTile;
          const int sk = seq % C::kKStages, sv = seq % C::kVStages;
          if (seq >= C::kKStages &&
              !mbar_wait(bar(C::kBarKEmpty + sk), (static_cast<uint32_t>(seq / C::kKStages) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::kBarKFull + sk), C::kTileBytes);
          tma_load_4d(base + C::kKOff + sk * C::kTileBytes, &p.tm_k, bar(C::kBarKFull + sk), 0, kv_row, g, b, pol_kv);
          if (seq >= C::kVStages &&
              !mbar_wait(bar(C::kBarVEmpty + sv), (static_cast<uint32_t>(seq / C::kVStages) & 1) ^ 1, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(bar(C::kBarVFull + sv), C::kTileBytes);
          tma_load_4d(base + C::kVOff + sv * C::kTileBytes, &p.tm_v, bar(C::kBarVFull + sv), 0, kv_row, g, b, pol_kv);
          ++seq;
        }
      }
      // let the copies still in flight land before the CTA can exit (matters only after an abort)
      for (int q = max(0, seq - C::kKStages); q < seq; ++q)
        mbar_wait_drain(bar(C::kBarKFull + q % C::kKStages), static_cast<uint32_t>(q / C::kKStages) & 1);
      for (int q = max(0, seq - C::kVStages); q < seq; ++q)
        mbar_wait_drain(bar(C::kBarVFull + q % C::kVStages), static_cast<uint32_t>(q / C::kVStages) & 1);
      mbar_wait_drain(bar(C::kBarQFull), 0);
    }
  } else if (warp == C::kWarpQK) {
    // ---------------------------------------------------------------- QK issuer
    if (lane == 0 && n_max > 0) {
      constexpr uint32_t idesc_qk = idesc_s8(128, 128);
      bool ok = mbar_wait(bar(C::kBarQFull), 0, abort_flag);
      int seq = 0;
      int prev_t = -1, prev_j = 0;  // reader of the S buffer's current contents
      for (int j = 0; ok && j < n_max; ++j) {
        for (int t = 0; ok && t < 2; ++t) {
          if (j >= (t ? n1 : n0)) continue;
          const int s = seq % C::kKStages;
          if (!mbar_wait(bar(C::kBarKFull + s), static_cast<uint32_t>(seq / C::kKStages) & 1, abort_flag) ||
              (prev_t >= 0 &&
               !mbar_wait(bar(C::kBarSFree + prev_t), static_cast<uint32_t>(prev_j) & 1, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qbase = base + C::kQOff + t * C::kTileBytes;
          const uint32_t kbase = base + C::kKOff + s * C::kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_i8_ss(tmem + C::kColS, sdesc_sw128(qbase + kk * 32, 16, 1024), sdesc_sw128(kbase + kk * 32, 16, 1024),
                      idesc_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::kBarSFull + t));
          mma_commit(bar(C::kBarKEmpty + s));
          qk_issued[t] = j + 1;  // lets the PV issuer queue behind this QK (see there)
          prev_t = t;
          prev_j = j;
          ++seq;
        }
      }
      // every MMA issued above has retired before TMEM can be released
      mma_commit(bar(C::kBarDrain));
      mbar_wait_drain(bar(C::kBarDrain), 0);
    }
  } else if (warp == C::kWarpPV) {
    // ---------------------------------------------------------------- PV issuer
    if (lane == 0 && n_max > 0) {
      constexpr uint32_t idesc_pv = idesc_e4m3(128, 144, true);
      const uint32_t ones = base + C::kOnesOff;
      bool ok = true;
      int seq = 0;
      for (int j = 0; ok && j < n_max; ++j) {
        for (int t = 0; ok && t < 2; ++t) {
          const int nt = t ? n1 : n0;
          if (j >= nt) continue;
          const int s = seq % C::kVStages;
          // QK_t(j+1) is on the softmax's critical path and this P·V is not (its P buffer is
          // reused only a block later): let that QK reach the tensor core first, as a single
          // issuer would order them (bounded; the order never affects results)
          if (j + 1 < nt) {
            for (int spin = 0; spin < 4096 && qk_issued[t] < j + 2 && !*abort_flag; ++spin) __nanosleep(32);
          }
          if (!mbar_wait(bar(C::kBarPFull + t), static_cast<uint32_t>(j) & 1, abort_flag) ||
              !mbar_wait(bar(C::kBarVFull + s), static_cast<uint32_t>(seq / C::kVStages) & 1, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t vbase = base + C::kVOff + s * C::kTileBytes;
          const uint32_t pcol = tmem + C::kColP + 32 * t;
          const uint32_t ocol = tmem + (t ? C::kColO1 : C::kColO0);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // 32 key rows per step: 8 TMEM columns of packed P8; B = 4096 B of V8 (MN atom 0)
            // and, one leading-byte offset further, the same 32 rows of the ones block (atom 1)
            const uint32_t vk = vbase + kk * 4096;
            mma_f8_ts(ocol, pcol + kk * 8, sdesc_sw128(vk, ones - vk, 1024), idesc_pv,
                      (j > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(bar(C::kBarPVDone + t));
          mma_commit(bar(C::kBarVEmpty + s));
          if (j == nt - 1) mma_commit(bar(C::kBarOFinal + t));
          ++seq;
        }
      }
      mma_commit(bar(C::kBarDrain + 1));
      mbar_wait_drain(bar(C::kBarDrain + 1), 0);
    }
  } else {
    // ---------------------------------------------------------------- softmax warps
    const int t = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int nt = t ? n1 : n0;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t i_glob = (int64_t)(2 * pr + t) * kTile + row;
    const float kNegInf = -__int_as_float(0x7f800000);
    const uint32_t s_col = tmem + lane_off + C::kColS;
    const uint32_t o_col = tmem + lane_off + (t ? C::kColO1 : C::kColO0);
    const uint32_t l_col = o_col + 128;
    const uint32_t p_col = tmem + lane_off + C::kColP + 32 * t;
    const uint16_t* list = lists + t * kQbsaMaxKBlocks;
    const float* ks_row = p.k_scale + ((int64_t)b * p.Nkv + g) * p.nkb;
    const float sq = (2 * pr + t < p.nqb ? p.q_scale[((int64_t)b * p.Nq + h) * p.nqb + 2 * pr + t] : 0.f);
    int kb_next = nt > 0 ? list[0] : 0;
    float ks_next = nt > 0 ? ks_row[kb_next] : 0.f;

    float m = kNegInf;    // running max, log2 domain
    float ref = kNegInf;  // power-of-two reference of the FP8 weights (an integer)
    // a last kept block that runs past S_kv is taken out of line after the loop
    const bool tail_last = nt > 0 && (p.Skv % kTile) != 0 && list[nt - 1] == p.nkb - 1;
    const int n_main = nt - (tail_last ? 1 : 0);
    bool ok = true;
    for (int j = 0; ok && j < n_main; ++j) {
      const float cst = (sq * ks_next) * p.scale_log2;
      if (j + 1 < nt) {  // the next block's key scale, fetched while this block is processed
        kb_next = list[j + 1];
        ks_next = ks_row[kb_next];
      }
      ok = warp_wait(bar(C::kBarSFull + t), static_cast<uint32_t>(j) & 1, abort_flag);
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[128];  // s32 scores; exact in f32 since |dot| <= 128 * 127^2 < 2^24
      tmem_ld128_wait(s_col, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarSFree + t));

      // row max of z = t * c: max(t) * c for c >= 0, min(t) * c otherwise (c is uniform)
      const bool pos = cst >= 0.f;
      const float m_blk = __int2float_rn(pos ? imax128(sv) : imin128(sv)) * cst;
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

      // p = 2^(t c - R) held in FP16 (the precision of P before its FP8 rounding),
      // then rounded to E4M3; four weights per packed word
      const uint64_t cc = pack_f32x2(cst, cst);
      const uint64_t nr = pack_f32x2(-ref, -ref);
      uint32_t pk[32];
#pragma unroll
      for (int x = 0; x < 32; ++x)
        pk[x] = i2f_fma_exp2_e4m3x4(sv[4 * x], sv[4 * x + 1], sv[4 * x + 2], sv[4 * x + 3], cc, nr);

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
            for (int x = 0; x < 32; ++x) rr[x] = __float_as_uint(__uint_as_float(rr[x]) * a);
            tmem_st32(o_col + ch * 32, rr);
          }
          tmem_st1(l_col, __float_as_uint(__uint_as_float(tmem_ld1_wait(l_col)) * a));
        }
      }
      tmem_st32(p_col, pk);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(C::kBarPFull + t));
    }
    if (ok && tail_last) {
      const int kb = kb_next;  // list[nt - 1]
      const QbsaTailResult r = qbsa_tail_block(s_col, o_col, p_col, bar(C::kBarSFull + t), bar(C::kBarSFree + t),
                                               bar(C::kBarPVDone + t), bar(C::kBarPFull + t), nt - 1,
                                               (sq * ks_next) * p.scale_log2, p.Skv - kb * kTile, m, ref, abort_flag);
      m = r.m;
      ref = r.ref;
      ok = r.ok != 0;
    }

    // ------------------------------------------------------------ epilogue
    bool have_o = ok && nt > 0;
    if (have_o) {
      // a dedicated single-use barrier: pv_done's parity cannot tell PV(n-1) from PV(n-3)
      have_o = warp_wait(bar(C::kBarOFinal + t), 0, abort_flag);
      tc_fence_after();
    }
    float l = 0.f;
    if (have_o) l = __uint_as_float(tmem_ld1_wait(l_col));
    const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
    const bool tile_live = 2 * pr + t < p.nqb;
    // O -> bf16: columns [0,64) staged in this tile's Q buffer (its last QK has retired),
    // columns [64,128) in a second buffer, both in the 128-byte-swizzled layout of the
    // output tensor map, then written by two TMA stores
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint32_t stage = hf ? base + C::kEOff + t * C::kTileBytes : base + C::kQOff + t * C::kTileBytes;
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
          const int c0 = hf * 64 + ch * 32 + 8 * x;
          float f[8];
#pragma unroll
          for (int y = 0; y < 8; ++y) f[y] = __uint_as_float(rr[8 * x + y]) * (vsc[c0 + y] * inv_l);
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
        tma_store_4d(&p.tm_o, base + C::kEOff + t * C::kTileBytes, 64, (2 * pr + t) * kTile, h, b);
        bulk_commit_group();
      }
      bulk_wait_read_all();  // shared memory must outlive the stores' reads
    }
    if (i_glob < p.Sq) {
      const int64_t sidx = ((int64_t)b * p.Nq + h) * p.Sq + i_glob;
      const bool live = l > 0.f;
      if (p.softmax_max) p.softmax_max[sidx] = live ? m * 0.6931471805599453f : kNegInf;
      if (p.softmax_sum) p.softmax_sum[sidx] = live ? l * ex2(ref - m) : 0.f;  // against the true max
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kWarpQK) {
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
  const uint8_t* row = mask + (int64_t)r * n_kb;
  const bool v16 = (n_kb % 16 == 0) && ((reinterpret_cast<uintptr_t>(mask) & 15u) == 0);
  const int cnt = v16 ? compact_mask_row_v16(row, n_kb, buf[warp], lane) : compact_mask_row(row, n_kb, buf[warp], lane);
  __syncwarp();
  for (int i = lane; i < n_kb; i += 32) lists[(int64_t)r * n_kb + i] = (i < cnt) ? buf[warp][i] : -1;
  if (lane == 0) counts[r] = cnt;
}

}  // namespace qbsa
