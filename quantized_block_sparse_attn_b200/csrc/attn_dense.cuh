// Dense bf16 fused attention forward for sm_100a.
//
// Computes Softmax(Mask(Q·Kᵀ·scale + pse))·V (npu_fusion_attention guide,
// "昇腾 NPU 融合注意力算子详解与迁移指南", §2 算子数学原理) one 128-row query tile per
// CTA, streaming 128-row K/V tiles with an online softmax so that the score matrix
// never reaches global memory (§2, the tiling remark).  Masks follow §4.2/§4.3,
// varlen TND follows §4.3, GQA follows §7, and the outputs are attention_out,
// softmax_max and softmax_sum (§5).  The unmasked D = 128 BNSD / BSND case goes to
// attn_pair_kernel (two query tiles per CTA, attn_pair.cuh); this kernel serves every
// other case, including bsa_fwd's block lists.
//
// CTA = 12 warps (three warpgroups).  After set-up the third warpgroup gives registers back
// (setmaxnreg, 168 -> 64 per thread) and the two softmax warpgroups take them (168 -> 216):
//   warps 0..7  softmax: query row 32*(warp%4)+lane (the warp's TMEM lane quarter);
//               warps 0..3 own score columns [0,64), warps 4..7 columns [64,128) of
//               the same rows, and exchange their partial row maxima through shared
//               memory (a 64-thread named barrier per lane quarter).  O is rescaled in
//               TMEM only when the running max grew by more than 2^8 (the lagging
//               reference cancels in O / l; the statistics are corrected at the end).
//               P goes to TMEM as bf16; the epilogue normalises O and stores it.
//   warp 8      TMA producer: Q once, then K/V tiles into a 2-stage ring each.
//   warp 9      MMA issuer (one thread): S = Q Kᵀ (kind::f16, SS) into a
//               double-buffered f32 TMEM tile, then O += P V (kind::f16, A = P from
//               TMEM, B = V from shared memory, MN-major).
//   warps 10-11 no work after set-up (warp 1 allocates and frees TMEM around the roles).
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) P0 [384,448) P1 [448,512).
//
// CTA order: query heads are taken in groups whose K/V fit in about 48 MB of L2; in
// a group the heaviest query tiles (causal) come first, heads fastest.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "ptx_sm100.cuh"
#include "schedule.cuh"

namespace qbsa {

constexpr int kMaxSeqs = 128;  // TND sequences per call (kernel-parameter tables, < 4 KB of params)

struct DenseParams {
  CUtensorMap tm_q;  // 4-D {D, rows, heads, batch}, box {64, 128, 1, 1}, bf16, SW128
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  __nv_bfloat16* out;
  float* softmax_max;
  float* softmax_sum;
  const uint8_t* atten_mask;   // 1 = masked; nullptr if none
  const __nv_bfloat16* pse;    // nullptr if none
  int64_t o_row_stride, o_head_stride, o_batch_stride;  // elements
  int64_t m_row_stride, m_head_stride, m_batch_stride;  // atten_mask strides (elements)
  int64_t p_row_stride, p_head_stride, p_batch_stride;  // pse strides (elements)
  int64_t stat_head_stride, stat_batch_stride;          // stats strides (elements)
  int64_t pre_tokens, next_tokens;
  int B, Nq, Nkv, Sq, Skv, group;
  int sparse_mode;
  int tnd;        // 1: varlen TND
  int n_qtiles;   // BNSD/BSND: ceil(Sq/128)
  int n_rank;     // query tiles per head (all batches / sequences)
  int head_grp;   // query heads per L2 group
  // optional 128x128 block mask [B, Nq, n_qtiles, mask_nkb] (1 = compute), BNSD / BSND only
  const uint8_t* block_mask;
  int mask_nkb;
  // atten_mask / pse tiles by TMA (rows 16-byte aligned: S_kv % 16 == 0 for the mask, % 8 for
  // pse, bases 16-byte aligned); otherwise the softmax warps read them element by element
  int mask_tma, pse_tma;
  int mask_heads, mask_batches;  // the mask's head / batch coordinates apply (B1SS, BNSS)
  int pse_batches;               // pse's batch coordinate applies (no batch broadcast)
  CUtensorMap tm_m;  // uint8 {S_kv, S_q, heads, batches}, box {128, 128, 1, 1}, SW128
  CUtensorMap tm_p;  // bf16 {S_kv, S_q, N_q, batches}, box {64, 128, 1, 1}, SW128
  float scale;
  // TND tables (sequences in processing order)
  int n_seq;
  int seq_q_start[kMaxSeqs];
  int seq_q_len[kMaxSeqs];
  int seq_kv_start[kMaxSeqs];
  int seq_kv_len[kMaxSeqs];
  int seq_tile_start[kMaxSeqs + 1];
};

template <int D>
struct DenseCfg {
  static constexpr int kStages = 2;
  static constexpr int kTileBytes = kTile * D * 2;  // one 128 x D bf16 tile
  static constexpr int kSubBytes = kTile * 128;     // one 128-row x 128-byte swizzle column
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kMOff = kVOff + kStages * kTileBytes;  // atten_mask tile, 128 x 128 bytes
  static constexpr int kPOff = kMOff + kTile * 128;             // pse tile, two 128 x 64 bf16 halves
  static constexpr int kXOff = kPOff + kTile * 256;             // row-max exchange: float [2][2][128]
  static constexpr int kListOff = kXOff + 2 * 2 * 128 * 4;    // uint16 kept K tiles (block mask)
  static constexpr int kMaxListed = 2048;
  static constexpr int kBarOff = kListOff + kMaxListed * 2;
  // barriers
  static constexpr int kBarQFull = 0;
  static constexpr int kBarKFull = 1;
  static constexpr int kBarKEmpty = kBarKFull + kStages;
  static constexpr int kBarVFull = kBarKEmpty + kStages;
  static constexpr int kBarVEmpty = kBarVFull + kStages;
  static constexpr int kBarSFull = kBarVEmpty + kStages;  // 2
  static constexpr int kBarSFree = kBarSFull + 2;         // 2
  static constexpr int kBarPFull = kBarSFree + 2;         // 2
  static constexpr int kBarPVDone = kBarPFull + 2;        // 1
  static constexpr int kBarOFinal = kBarPVDone + 1;       // 1: last P·V done (single use)
  static constexpr int kBarMFull = kBarOFinal + 1;        // 1: atten_mask / pse tile landed
  static constexpr int kBarMEmpty = kBarMFull + 1;        // 1: ... and read by every softmax thread
  static constexpr int kNumBars = kBarMEmpty + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  // + alignment slack; at least 120 KB so that one CTA holds an SM (and its 512 TMEM columns)
  static constexpr int kSmemUsed = kMiscOff + 16 + 1024;
  static constexpr int kSmemBytes = kSmemUsed > 120 * 1024 ? kSmemUsed : 120 * 1024;
  // TMEM columns
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP0 = 384, kColP1 = 448;
  static constexpr int kThreads = 384;
  static constexpr int kSoftmaxThreads = 256;
};
static_assert(DenseCfg<128>::kSmemBytes <= 232448, "shared memory above the 227 KB opt-in limit");
static_assert(DenseCfg<128>::kMOff % 1024 == 0 && DenseCfg<64>::kMOff % 1024 == 0,
              "swizzled buffers must start on 1024-byte boundaries");
constexpr int kDenseRegSoftmax = 216, kDenseRegHelper = 64;  // per thread, after set-up
static_assert(2 * 128 * kDenseRegSoftmax + 128 * kDenseRegHelper <= 384 * 168,
              "register shares above what a 168-register launch holds");

struct DenseWork {
  int b, h, qt;
  int64_t q_row0;   // tensor-map row coordinate of query row 0 of the tile's sequence
  int64_t kv_row0;  // tensor-map row coordinate of key row 0 of the sequence
  int coord_b;      // tensor-map batch coordinate
  int64_t sq, skv;  // sequence lengths
  int64_t tok0;     // TND: first token of the sequence (stats / output addressing)
};

__device__ __forceinline__ DenseWork dense_work(const DenseParams& p) {
  DenseWork w;
  // head groups (L2 reuse of K/V), heaviest query tiles first, heads fastest inside a group
  const int64_t per_group = (int64_t)p.head_grp * p.n_rank;
  const int grp = static_cast<int>(blockIdx.x / per_group);
  const int h0 = grp * p.head_grp;
  const int hcount = min(p.head_grp, p.Nq - h0);
  const int off = static_cast<int>(blockIdx.x - grp * per_group);
  const int r = off / hcount;
  w.h = h0 + off % hcount;
  if (!p.tnd) {
    const int rank = r / p.B;
    w.b = r % p.B;
    w.qt = p.n_qtiles - 1 - rank;
    w.q_row0 = 0;
    w.kv_row0 = 0;
    w.coord_b = w.b;
    w.sq = p.Sq;
    w.skv = p.Skv;
    w.tok0 = 0;
  } else {
    int lo = 0, hi = p.n_seq - 1;
    while (lo < hi) {  // last i with seq_tile_start[i] <= r
      const int mid = (lo + hi + 1) >> 1;
      if (p.seq_tile_start[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int ntile = p.seq_tile_start[lo + 1] - p.seq_tile_start[lo];
    w.b = lo;  // index in processing order (tables are already permuted)
    w.qt = ntile - 1 - (r - p.seq_tile_start[lo]);
    w.q_row0 = p.seq_q_start[lo];
    w.kv_row0 = p.seq_kv_start[lo];
    w.coord_b = 0;
    w.sq = p.seq_q_len[lo];
    w.skv = p.seq_kv_len[lo];
    w.tok0 = p.seq_q_start[lo];
  }
  return w;
}

// Word k (0..3, a compile-time index after unrolling) of a 16-byte vector.
__device__ __forceinline__ uint32_t u4_word(const uint4& v, int k) {
  return k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
}

// kGeneral: an explicit atten_mask or pse is present (the instantiation without them carries
// none of their code, which the other callers would otherwise pay for in the softmax loop).
template <int D, bool kGeneral>
__global__ void __launch_bounds__(384, 1) attn_dense_kernel(const __grid_constant__ DenseParams p) {
  using C = DenseCfg<D>;
  constexpr int kHalfD = D / 2;  // O columns per softmax half
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
  float* xch = reinterpret_cast<float*>(smem + C::kXOff);  // [slot][half][row]

  const DenseWork w = dense_work(p);
  const int g = w.h / p.group;
  const Band band = band_of(p.sparse_mode, p.pre_tokens, p.next_tokens, w.sq, w.skv);
  const TileRange tr = tile_range(w.qt, w.sq, w.skv, band);
  constexpr bool general_mask = kGeneral;
  uint16_t* klist = reinterpret_cast<uint16_t*>(smem + C::kListOff);
  int* count_slot = reinterpret_cast<int*>(smem + C::kMiscOff + 8);

  if (p.block_mask != nullptr && warp == 0) {
    // kept K tiles of this query tile inside its band range, ascending
    const uint8_t* mrow = p.block_mask + (((int64_t)w.b * p.Nq + w.h) * p.n_qtiles + w.qt) * p.mask_nkb;
    int cnt = 0;
    for (int j0 = tr.kt_begin; j0 < tr.kt_end; j0 += 32) {
      const int j = j0 + lane;
      const bool keep = (j < tr.kt_end) && (mrow[j] != 0);
      const uint32_t bal = __ballot_sync(0xffffffffu, keep);
      if (keep) klist[cnt + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(j);
      cnt += __popc(bal);
    }
    if (lane == 0) *count_slot = cnt;
  }
  if (threadIdx.x == 0) {
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
    mbar_init(bar(C::kBarMFull), 1);
    mbar_init(bar(C::kBarMEmpty), C::kSoftmaxThreads);
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_q);
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
    if (kGeneral && p.mask_tma) tma_prefetch_desc(&p.tm_m);
    if (kGeneral && p.pse_tma) tma_prefetch_desc(&p.tm_p);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool listed = p.block_mask != nullptr;
  const int n = listed ? *count_slot : tr.kt_end - tr.kt_begin;
  auto ktile = [&](int it) -> int { return listed ? static_cast<int>(klist[it]) : tr.kt_begin + it; };

  if (warp >= 8) {
    regs_dec<kDenseRegHelper>();
    if (warp == 8) {
      // ---------------------------------------------------------------- producer
      if (lane == 0 && n > 0) {
        const uint64_t pol_q = l2_policy_evict_first();
        const uint64_t pol_kv = l2_policy_evict_last();
        const int q_row = static_cast<int>(w.q_row0 + (int64_t)w.qt * kTile);
        int n_staged = 0;  // atten_mask / pse tiles loaded
        mbar_arrive_expect_tx(bar(C::kBarQFull), C::kTileBytes);
        for (int sub = 0; sub < D / 64; ++sub)
          tma_load_4d(base + C::kQOff + sub * C::kSubBytes, &p.tm_q, bar(C::kBarQFull), sub * 64, q_row, w.h,
                      w.coord_b, pol_q);
        for (int it = 0; it < n; ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1;
          const int kv_row = static_cast<int>(w.kv_row0 + (int64_t)ktile(it) * kTile);
          if (it >= C::kStages && !mbar_wait(bar(C::kBarKEmpty + s), ph ^ 1, abort_flag)) break;
          mbar_arrive_expect_tx(bar(C::kBarKFull + s), C::kTileBytes);
          for (int sub = 0; sub < D / 64; ++sub)
            tma_load_4d(base + C::kKOff + s * C::kTileBytes + sub * C::kSubBytes, &p.tm_k, bar(C::kBarKFull + s),
                        sub * 64, kv_row, g, w.coord_b, pol_kv);
          if (it >= C::kStages && !mbar_wait(bar(C::kBarVEmpty + s), ph ^ 1, abort_flag)) break;
          mbar_arrive_expect_tx(bar(C::kBarVFull + s), C::kTileBytes);
          for (int sub = 0; sub < D / 64; ++sub)
            tma_load_4d(base + C::kVOff + s * C::kTileBytes + sub * C::kSubBytes, &p.tm_v, bar(C::kBarVFull + s),
                        sub * 64, kv_row, g, w.coord_b, pol_kv);
          if (kGeneral && (p.mask_tma || p.pse_tma)) {
            // atten_mask / pse tile of (query tile, key tile) into the single-stage buffer, once
            // every softmax thread has read the previous one (early in its step, so the load has
            // about a step to land)
            if (it >= 1 && !mbar_wait(bar(C::kBarMEmpty), (it - 1) & 1, abort_flag)) break;
            const int kc = ktile(it) * kTile, qr = w.qt * kTile;
            mbar_arrive_expect_tx(bar(C::kBarMFull), (p.mask_tma ? kTile * 128 : 0) + (p.pse_tma ? kTile * 256 : 0));
            if (p.mask_tma)  // shared by heads (and batches) for SS / B1SS: keep it in L2
              tma_load_4d(base + C::kMOff, &p.tm_m, bar(C::kBarMFull), kc, qr, p.mask_heads ? w.h : 0,
                          p.mask_batches ? w.b : 0, pol_kv);
            if (p.pse_tma) {
              for (int hf = 0; hf < 2; ++hf)
                tma_load_4d(base + C::kPOff + hf * kTile * 128, &p.tm_p, bar(C::kBarMFull), kc + 64 * hf, qr, w.h,
                            p.pse_batches ? w.b : 0, pol_q);
            }
            n_staged = it + 1;
          }
        }
        // the last staged tile has landed before the CTA can exit (matters only after an abort)
        if (n_staged > 0) mbar_wait_drain(bar(C::kBarMFull), static_cast<uint32_t>(n_staged - 1) & 1);
      }
    } else if (warp == 9) {
      // ---------------------------------------------------------------- MMA issuer
      if (lane == 0 && n > 0) {
        constexpr uint32_t idesc_qk = idesc_bf16(128, 128, false);
        constexpr uint32_t idesc_pv = idesc_bf16(128, D, true);
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
          for (int kk = 0; kk < kTile / 16; ++kk) {
            // B = V tile, MN-major: 16 key rows per step (2048 B), D-halves 16 KB apart
            const uint64_t bdesc = sdesc_sw128(vbase + kk * 2048, C::kSubBytes, 1024);
            mma_f16_ts(tmem + C::kColO, tmem + pcol + kk * 8, bdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
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
          for (int kk = 0; kk < D / 16; ++kk) {
            // A = Q, B = K, both K-major: 16 elements (32 B) per step inside a 64-wide column
            const uint32_t off = (kk >> 2) * C::kSubBytes + (kk & 3) * 32;
            mma_f16_ss(tmem + scol, sdesc_sw128(qbase + off, 16, 1024), sdesc_sw128(kbase + off, 16, 1024), idesc_qk,
                       kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::kBarSFull + bi));
          mma_commit(bar(C::kBarKEmpty + s));
          if (it >= 1 && !issue_pv(it - 1)) { ok = false; break; }
        }
        if (ok && issue_pv(n - 1)) mma_commit(bar(C::kBarOFinal));
      }
    }
  } else {
    regs_inc<kDenseRegSoftmax>();
    // ---------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int half = warp >> 2;  // 0: score columns [0,64), 1: [64,128)
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int64_t i_loc = (int64_t)w.qt * kTile + row;  // query index inside the sequence
    const bool has_pse = kGeneral && p.pse != nullptr;
    const float vs = has_pse ? 1.0f : p.scale;  // score = value * vs
    const float c = vs * 1.4426950408889634f;   // value -> log2 domain
    const float kNegInf = -__int_as_float(0x7f800000);
    const int64_t j_lo = i_loc - band.lo_off;   // per-row band, column indices of the sequence
    const int64_t j_hi = min64(w.skv - 1, i_loc + band.hi_off);
    const uint32_t o_col = tmem + lane_off + C::kColO + half * kHalfD;

    const uint8_t* mrow = nullptr;
    const __nv_bfloat16* prow = nullptr;
    if (kGeneral && p.atten_mask && i_loc < w.sq)
      mrow = p.atten_mask + w.b * p.m_batch_stride + w.h * p.m_head_stride + i_loc * p.m_row_stride;
    if (has_pse && i_loc < w.sq)
      prow = p.pse + w.b * p.p_batch_stride + w.h * p.p_head_stride + i_loc * p.p_row_stride;

    // atten_mask / pse of a key tile: staged by the producer (TMA, 128-byte swizzle: 16-byte
    // chunk c of row r sits at chunk c ^ (r % 8)), this row's 64 mask bytes / 64 pse values of
    // the half read as four / eight 16-byte loads; without TMA (unaligned rows) read element by
    // element from global memory
    const bool m_tma = kGeneral && p.mask_tma, p_tma = kGeneral && p.pse_tma;
    const uint32_t m_line = base + C::kMOff + row * 128;
    const uint32_t p_line = base + C::kPOff + half * (kTile * 128) + row * 128;
    const uint32_t swz = static_cast<uint32_t>(row & 7);

    float m_ref = kNegInf, m_true = kNegInf, l = 0.f;  // l: this half's partial sum
    bool ok = true;
    for (int it = 0; it < n; ++it) {
      const int kt = ktile(it);
      const int bi = it & 1;
      // never leave the loop early: the paired warp waits on named barriers below, so
      // after a failed (timed-out) wait the remaining iterations run without waiting
      if (ok) ok = mbar_wait(bar(C::kBarSFull + bi), (it >> 1) & 1, abort_flag);
      tc_fence_after();
      float sv[64];
      {
        uint32_t r[64];
        tmem_ld64_wait(tmem + lane_off + (bi ? C::kColS1 : C::kColS0) + half * 64, r);
#pragma unroll
        for (int x = 0; x < 64; ++x) sv[x] = __uint_as_float(r[x]);
      }
      tc_fence_before();
      mbar_arrive(bar(C::kBarSFree + bi));

      const bool full = (kt >= tr.full_begin && kt < tr.full_end);
      if (!full || general_mask) {
        const int64_t col0 = (int64_t)kt * kTile + half * 64;
        const int64_t clo = j_lo - col0, chi = j_hi - col0;
        if (kGeneral && (m_tma || p_tma)) {
          if (ok) ok = mbar_wait(bar(C::kBarMFull), static_cast<uint32_t>(it) & 1, abort_flag);
        }
        if (kGeneral && has_pse) {
          if (p_tma) {
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8) {
              const uint4 v8 = lds128(p_line + ((static_cast<uint32_t>(c8) ^ swz) << 4));
#pragma unroll
              for (int y = 0; y < 8; ++y) {
                const int x = 8 * c8 + y;
                const uint32_t wd = u4_word(v8, y >> 1);
                sv[x] = sv[x] * p.scale + __uint_as_float((y & 1) ? (wd & 0xffff0000u) : (wd << 16));
              }
            }
          } else {
#pragma unroll
            for (int x = 0; x < 64; ++x) {
              const int64_t j = col0 + x;
              sv[x] = sv[x] * p.scale + ((prow && j < w.skv) ? __bfloat162float(prow[j]) : 0.f);
            }
          }
        }
        uint32_t nz[16];  // bit 8k+7 of nz[i]: mask byte 4i+k of this half is nonzero (masked)
        if (m_tma) {
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint4 v4 = lds128(m_line + ((static_cast<uint32_t>(4 * half + c4) ^ swz) << 4));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t wd = u4_word(v4, k);
              nz[4 * c4 + k] = (((wd & 0x7f7f7f7fu) + 0x7f7f7f7fu) | wd) & 0x80808080u;
            }
          }
        }
        if (kGeneral && (m_tma || p_tma)) mbar_arrive(bar(C::kBarMEmpty));  // this thread is done with the tile
        if (m_tma) {
          if (clo <= 0 && chi >= 63) {  // the whole half lies inside this row's band
#pragma unroll
            for (int x = 0; x < 64; ++x)
              sv[x] = ((nz[x >> 2] >> (8 * (x & 3) + 7)) & 1u) ? kNegInf : sv[x];
          } else {
#pragma unroll
            for (int x = 0; x < 64; ++x) {
              const bool keep = (x >= clo) && (x <= chi) && !((nz[x >> 2] >> (8 * (x & 3) + 7)) & 1u);
              sv[x] = keep ? sv[x] : kNegInf;
            }
          }
        } else if (kGeneral && mrow) {
#pragma unroll
          for (int x = 0; x < 64; ++x) {
            const int64_t j = col0 + x;
            const bool keep = (x >= clo) && (x <= chi) && (j < w.skv) && (mrow[j] == 0);
            sv[x] = keep ? sv[x] : kNegInf;
          }
        } else if (!(clo <= 0 && chi >= 63)) {  // band only, and the half is not inside it
#pragma unroll
          for (int x = 0; x < 64; ++x) sv[x] = (x >= clo && x <= chi) ? sv[x] : kNegInf;
        }
      }
      const float pmax = max64(sv);
      // combine the two halves of the row
      float* slot = xch + (it & 1) * 256;
      slot[half * 128 + row] = pmax;
      named_bar_sync(1 + quarter, 64);
      const float rmax = fmaxf(pmax, slot[(half ^ 1) * 128 + row]);

      const float m_new = fmaxf(m_true, rmax);
      const bool upd = (m_new > m_ref) && (m_ref == kNegInf || (m_new - m_ref) * c > 8.0f);
      const float alpha = upd ? ex2((m_ref - m_new) * c) : 1.0f;
      const bool need = upd && (it > 0) && (m_ref != kNegInf);
      if (__any_sync(0xffffffffu, need)) {
        // rescale this half of O: PV(it-1) must be complete first
        if (ok) ok = mbar_wait(bar(C::kBarPVDone), (it - 1) & 1, abort_flag);
        tc_fence_after();
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < kHalfD / 32; ++ch) {
          tmem_ld32_wait(o_col + ch * 32, r);
#pragma unroll
          for (int x = 0; x < 32; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
          tmem_st32(o_col + ch * 32, r);
        }
        tmem_st_wait();
      }
      if (upd) {
        l *= alpha;
        m_ref = m_new;
      }
      m_true = m_new;
      const float mc = (m_ref == kNegInf) ? 0.f : m_ref * c;
      uint32_t pk[32];
      float ls[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums (short dependency chains)
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const float p0 = ex2(fmaf(sv[2 * x], c, -mc));
        const float p1 = ex2(fmaf(sv[2 * x + 1], c, -mc));
        ls[x & 3] += p0 + p1;
        pk[x] = pack_bf16x2(p0, p1);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      tmem_st32(tmem + lane_off + (bi ? C::kColP1 : C::kColP0) + half * 32, pk);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(C::kBarPFull + bi));
    }

    // ------------------------------------------------------------ epilogue
    // total row sum: exchange the two halves' partial sums (slot n&1 was last read at n-2)
    {
      float* slot = xch + (n & 1) * 256;
      slot[half * 128 + row] = l;
      named_bar_sync(1 + quarter, 64);
      l += slot[(half ^ 1) * 128 + row];
    }
    const bool row_valid = i_loc < w.sq;
    bool have_o = ok && n > 0;
    if (have_o) {
      // a dedicated single-use barrier: pv_done's parity cannot tell PV(n-1) from PV(n-3)
      have_o = mbar_wait(bar(C::kBarOFinal), 0, abort_flag);
      tc_fence_after();
    }
    const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
    __nv_bfloat16* orow = nullptr;
    if (row_valid) {
      const int64_t orow_idx = p.tnd ? (w.tok0 + i_loc) : i_loc;
      orow = p.out + (p.tnd ? 0 : (int64_t)w.b * p.o_batch_stride) + (int64_t)w.h * p.o_head_stride +
             orow_idx * p.o_row_stride + half * kHalfD;
    }
#pragma unroll
    for (int ch = 0; ch < kHalfD / 32; ++ch) {
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
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * x + 0]) * inv_l, __uint_as_float(r[8 * x + 1]) * inv_l);
          v.y = pack_bf16x2(__uint_as_float(r[8 * x + 2]) * inv_l, __uint_as_float(r[8 * x + 3]) * inv_l);
          v.z = pack_bf16x2(__uint_as_float(r[8 * x + 4]) * inv_l, __uint_as_float(r[8 * x + 5]) * inv_l);
          v.w = pack_bf16x2(__uint_as_float(r[8 * x + 6]) * inv_l, __uint_as_float(r[8 * x + 7]) * inv_l);
          dst[x] = v;
        }
      }
    }
    if (half == 0 && row_valid && (p.softmax_max || p.softmax_sum)) {
      const int64_t sidx = p.tnd ? ((int64_t)w.h * p.stat_head_stride + w.tok0 + i_loc)
                                 : ((int64_t)w.b * p.stat_batch_stride + (int64_t)w.h * p.stat_head_stride + i_loc);
      const bool live = (m_true != kNegInf) && (l > 0.f);
      const float smax = live ? m_true * vs : kNegInf;
      const float ssum = live ? l * ex2((m_ref - m_true) * c) : 0.f;
      if (p.softmax_max) p.softmax_max[sidx] = smax;
      if (p.softmax_sum) p.softmax_sum[sidx] = ssum;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace qbsa
