// C ABI of libqbsa.so: argument validation, TMA tensor maps and kernel launches.
// The contract of every entry point is documented in include/qbsa.h.
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <numeric>
#include <string>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/qbsa.h"
#include "attn_dense.cuh"
#include "attn_pair.cuh"
#include "attn_pair_masked.cuh"
#include "attn_qbsa.cuh"
#include "estimate.cuh"
#include "quantize.cuh"
#include "schedule.cuh"

namespace {

thread_local std::string g_last_error;

qbsa_status fail(qbsa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

qbsa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(QBSA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t kTokenClamp = (int64_t)1 << 40;  // |pre/next| beyond this act as unbounded
constexpr int64_t kMaxLen = ((int64_t)1 << 31) - 256;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

qbsa_status get_encoder(EncodeTiledFn* out) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
      return fail(QBSA_ERR_CUDA, "cuTensorMapEncodeTiled is not available (%s)", cudaGetErrorString(e));
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  *out = fn;
  return QBSA_OK;
}

// 4-D tiled map over {inner, rows, heads, batch} with a {box0, 128, 1, 1} box and
// 128-byte swizzle.  strides[] are the byte strides of dims 1..3.
qbsa_status make_map(CUtensorMap* map, CUtensorMapDataType dt, const void* ptr, const uint64_t dims[4],
                     const uint64_t strides[3], uint32_t box0) {
  EncodeTiledFn enc;
  qbsa_status st = get_encoder(&enc);
  if (st != QBSA_OK) return st;
  cuuint64_t gd[4] = {dims[0], dims[1], dims[2], dims[3]};
  cuuint64_t gs[3] = {strides[0], strides[1], strides[2]};
  cuuint32_t box[4] = {box0, 128, 1, 1};
  cuuint32_t es[4] = {1, 1, 1, 1};
  CUresult r = enc(map, dt, 4, const_cast<void*>(ptr), gd, gs, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(QBSA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d; dims %llu %llu %llu %llu)", (int)r,
                (unsigned long long)dims[0], (unsigned long long)dims[1], (unsigned long long)dims[2],
                (unsigned long long)dims[3]);
  return QBSA_OK;
}

// Query heads per CTA group so that the group's K/V (kv_bytes_per_qhead each) stay in
// roughly 48 MB of the 126 MB L2 while the group's CTAs run.
int head_group(double kv_bytes_per_qhead, int n_heads) {
  const double budget = 48.0 * 1024 * 1024;
  int g = static_cast<int>(budget / std::max(kv_bytes_per_qhead, 1.0));
  return std::max(1, std::min(g, n_heads));
}

template <typename K>
qbsa_status set_smem(K kernel, int bytes) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
  return QBSA_OK;
}

qbsa_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return QBSA_OK;
}

// ------------------------------------------------------------------------------
// attn_fwd
// ------------------------------------------------------------------------------

struct SeqInfo {
  int q_start, q_len, kv_start, kv_len;
};

template <int D, bool kGeneral>
qbsa_status launch_dense_as(qbsa::DenseParams& prm, int64_t n_work, cudaStream_t stream) {
  using C = qbsa::DenseCfg<D>;
  qbsa_status st = set_smem(qbsa::attn_dense_kernel<D, kGeneral>, C::kSmemBytes);
  if (st != QBSA_OK) return st;
  qbsa::attn_dense_kernel<D, kGeneral>
      <<<dim3(static_cast<unsigned>(n_work)), C::kThreads, C::kSmemBytes, stream>>>(prm);
  return check_launch("attn_dense_kernel launch");
}

template <int D>
qbsa_status launch_dense(qbsa::DenseParams& prm, int64_t n_work, cudaStream_t stream) {
  const bool general = prm.atten_mask != nullptr || prm.pse != nullptr;
  return general ? launch_dense_as<D, true>(prm, n_work, stream) : launch_dense_as<D, false>(prm, n_work, stream);
}

}  // namespace

extern "C" {

int qbsa_version(void) { return 103; }

const char* qbsa_last_error(void) { return g_last_error.c_str(); }

// attn_fwd, optionally restricted to the 128x128 blocks kept by block_mask (bsa_fwd).
static qbsa_status attn_fwd_impl(const void* q, const void* k, const void* v, int B, int Nq, int Nkv, int Sq, int Skv,
                                 int D, int head_num, qbsa_layout input_layout, const uint8_t* atten_mask,
                                 qbsa_mask_shape mask_shape, const void* pse, int pse_batch_bcast, float scale,
                                 float keep_prob, int sparse_mode, int64_t pre_tokens, int64_t next_tokens,
                                 const int64_t* actual_seq_qlen, const int64_t* actual_seq_kvlen,
                                 void* attention_out, float* softmax_max, float* softmax_sum, void* stream,
                                 const uint8_t* block_mask) {
  // ---------------------------------------------------------------- validation
  if (!q || !k || !v || !attention_out) return fail(QBSA_ERR_INVALID, "q, k, v and attention_out must be non-null");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(attention_out))
    return fail(QBSA_ERR_INVALID, "q, k, v and attention_out must be 16-byte aligned");
  if ((softmax_max && !aligned16(softmax_max)) || (softmax_sum && !aligned16(softmax_sum)))
    return fail(QBSA_ERR_INVALID, "softmax_max / softmax_sum must be 16-byte aligned");
  if (B < 1 || Nq < 1 || Nkv < 1 || Sq < 0 || Skv < 0) return fail(QBSA_ERR_INVALID, "B, Nq, Nkv >= 1 and Sq, Skv >= 0");
  if (Sq > kMaxLen || Skv > kMaxLen) return fail(QBSA_ERR_UNSUPPORTED, "sequence length above %lld", (long long)kMaxLen);
  if (head_num != Nq) return fail(QBSA_ERR_INVALID, "head_num (%d) must equal Nq (%d)", head_num, Nq);
  if (Nq % Nkv != 0) return fail(QBSA_ERR_INVALID, "Nq (%d) must be a multiple of Nkv (%d)", Nq, Nkv);
  if (D < 1 || D > 768) return fail(QBSA_ERR_INVALID, "D must be in [1, 768]");
  if (D != 64 && D != 128) return fail(QBSA_ERR_UNSUPPORTED, "this build supports D = 64 or 128 (got %d)", D);
  if (input_layout != QBSA_LAYOUT_BNSD && input_layout != QBSA_LAYOUT_BSND && input_layout != QBSA_LAYOUT_TND)
    return fail(QBSA_ERR_INVALID, "unknown input_layout %d", (int)input_layout);
  if (!std::isfinite(scale)) return fail(QBSA_ERR_INVALID, "scale must be finite");
  if (!(keep_prob > 0.f && keep_prob <= 1.f)) return fail(QBSA_ERR_INVALID, "keep_prob must be in (0, 1]");
  if (keep_prob != 1.f) return fail(QBSA_ERR_UNSUPPORTED, "dropout (keep_prob < 1) is not implemented");
  if (sparse_mode != 0 && sparse_mode != 2 && sparse_mode != 3)
    return fail(QBSA_ERR_UNSUPPORTED, "sparse_mode %d is not implemented (0, 2, 3 are)", sparse_mode);
  if (mask_shape < QBSA_MASK_NONE || mask_shape > QBSA_MASK_BNSS)
    return fail(QBSA_ERR_INVALID, "unknown mask_shape %d", (int)mask_shape);
  if ((atten_mask == nullptr) != (mask_shape == QBSA_MASK_NONE))
    return fail(QBSA_ERR_INVALID, "atten_mask must be given exactly when mask_shape != QBSA_MASK_NONE");
  const bool tnd = input_layout == QBSA_LAYOUT_TND;
  if (tnd && (atten_mask || pse)) return fail(QBSA_ERR_UNSUPPORTED, "atten_mask / pse with TND is not implemented");
  if (tnd && (!actual_seq_qlen || !actual_seq_kvlen))
    return fail(QBSA_ERR_INVALID, "TND needs actual_seq_qlen and actual_seq_kvlen");
  if (!tnd && (actual_seq_qlen || actual_seq_kvlen))
    return fail(QBSA_ERR_INVALID, "actual_seq_qlen / actual_seq_kvlen are for TND only");
  if (tnd && B > qbsa::kMaxSeqs) return fail(QBSA_ERR_UNSUPPORTED, "TND supports at most %d sequences", qbsa::kMaxSeqs);
  if (pse && !aligned16(pse)) return fail(QBSA_ERR_INVALID, "pse must be 16-byte aligned");

  std::vector<SeqInfo> seqs;
  if (tnd) {
    int64_t pq = 0, pk = 0;
    for (int b = 0; b < B; ++b) {
      const int64_t cq = actual_seq_qlen[b], ck = actual_seq_kvlen[b];
      if (cq < pq || ck < pk) return fail(QBSA_ERR_INVALID, "actual_seq_*len must be non-decreasing cumulative sums");
      seqs.push_back({(int)pq, (int)(cq - pq), (int)pk, (int)(ck - pk)});
      pq = cq;
      pk = ck;
    }
    if (pq != Sq || pk != Skv)
      return fail(QBSA_ERR_INVALID, "last actual_seq_qlen/kvlen (%lld, %lld) must equal Sq/Skv (%d, %d)",
                  (long long)pq, (long long)pk, Sq, Skv);
  }
  if (Sq == 0) return QBSA_OK;  // nothing to compute

  const int64_t pre = std::max(-kTokenClamp, std::min(kTokenClamp, pre_tokens));
  const int64_t nxt = std::max(-kTokenClamp, std::min(kTokenClamp, next_tokens));

  // ---------------------------------------------------------------- parameters
  qbsa::DenseParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.out = static_cast<__nv_bfloat16*>(attention_out);
  prm.softmax_max = softmax_max;
  prm.softmax_sum = softmax_sum;
  prm.B = B;
  prm.Nq = Nq;
  prm.Nkv = Nkv;
  prm.Sq = Sq;
  prm.Skv = Skv;
  prm.group = Nq / Nkv;
  prm.sparse_mode = sparse_mode;
  prm.pre_tokens = pre;
  prm.next_tokens = nxt;
  prm.scale = scale;
  prm.tnd = tnd ? 1 : 0;
  const int64_t eD = D;
  uint64_t qd[4], kd[4], qs[3], ks[3];
  if (input_layout == QBSA_LAYOUT_BNSD) {
    prm.o_row_stride = eD;
    prm.o_head_stride = (int64_t)Sq * eD;
    prm.o_batch_stride = (int64_t)Nq * Sq * eD;
    qd[0] = D; qd[1] = Sq; qd[2] = Nq; qd[3] = B;
    kd[0] = D; kd[1] = Skv; kd[2] = Nkv; kd[3] = B;
    qs[0] = eD * 2; qs[1] = (uint64_t)Sq * eD * 2; qs[2] = (uint64_t)Nq * Sq * eD * 2;
    ks[0] = eD * 2; ks[1] = (uint64_t)Skv * eD * 2; ks[2] = (uint64_t)Nkv * Skv * eD * 2;
  } else if (input_layout == QBSA_LAYOUT_BSND) {
    prm.o_row_stride = (int64_t)Nq * eD;
    prm.o_head_stride = eD;
    prm.o_batch_stride = (int64_t)Sq * Nq * eD;
    qd[0] = D; qd[1] = Sq; qd[2] = Nq; qd[3] = B;
    kd[0] = D; kd[1] = Skv; kd[2] = Nkv; kd[3] = B;
    qs[0] = (uint64_t)Nq * eD * 2; qs[1] = eD * 2; qs[2] = (uint64_t)Sq * Nq * eD * 2;
    ks[0] = (uint64_t)Nkv * eD * 2; ks[1] = eD * 2; ks[2] = (uint64_t)Skv * Nkv * eD * 2;
  } else {
    prm.o_row_stride = (int64_t)Nq * eD;
    prm.o_head_stride = eD;
    prm.o_batch_stride = 0;
    qd[0] = D; qd[1] = Sq; qd[2] = Nq; qd[3] = 1;
    kd[0] = D; kd[1] = std::max(Skv, 1); kd[2] = Nkv; kd[3] = 1;
    qs[0] = (uint64_t)Nq * eD * 2; qs[1] = eD * 2; qs[2] = (uint64_t)Sq * Nq * eD * 2;
    ks[0] = (uint64_t)Nkv * eD * 2; ks[1] = eD * 2; ks[2] = (uint64_t)std::max(Skv, 1) * Nkv * eD * 2;
  }
  if (!tnd && Skv == 0) kd[1] = 1;  // map needs a non-zero extent; no tile is visited
  if (tnd) {
    prm.stat_head_stride = Sq;
    prm.stat_batch_stride = 0;
  } else {
    prm.stat_head_stride = Sq;
    prm.stat_batch_stride = (int64_t)Nq * Sq;
  }
  if (atten_mask) {
    prm.atten_mask = atten_mask;
    prm.m_row_stride = Skv;
    prm.m_head_stride = (mask_shape == QBSA_MASK_BNSS) ? (int64_t)Sq * Skv : 0;
    prm.m_batch_stride = (mask_shape == QBSA_MASK_SS) ? 0
                         : (mask_shape == QBSA_MASK_B1SS) ? (int64_t)Sq * Skv
                                                          : (int64_t)Nq * Sq * Skv;
  }
  if (pse) {
    prm.pse = static_cast<const __nv_bfloat16*>(pse);
    prm.p_row_stride = Skv;
    prm.p_head_stride = (int64_t)Sq * Skv;
    prm.p_batch_stride = pse_batch_bcast ? 0 : (int64_t)Nq * Sq * Skv;
  }

  int64_t n_rank = 0;
  if (tnd) {
    std::vector<int> order(B);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b2) { return seqs[a].q_len > seqs[b2].q_len; });
    prm.n_seq = B;
    int acc = 0;
    for (int i = 0; i < B; ++i) {
      const SeqInfo& s = seqs[order[i]];
      prm.seq_q_start[i] = s.q_start;
      prm.seq_q_len[i] = s.q_len;
      prm.seq_kv_start[i] = s.kv_start;
      prm.seq_kv_len[i] = s.kv_len;
      prm.seq_tile_start[i] = acc;
      acc += (s.q_len + qbsa::kTile - 1) / qbsa::kTile;
    }
    prm.seq_tile_start[B] = acc;
    n_rank = acc;
  } else {
    prm.n_qtiles = (Sq + qbsa::kTile - 1) / qbsa::kTile;
    n_rank = (int64_t)prm.n_qtiles * B;
  }
  const int64_t n_work = n_rank * Nq;
  if (n_work == 0) return QBSA_OK;
  if (n_work > 0x7fffffffLL) return fail(QBSA_ERR_UNSUPPORTED, "too many query tiles (%lld)", (long long)n_work);
  prm.n_rank = static_cast<int>(n_rank);
  // K/V bytes of one query head: one kv head (all batches; all sequences for TND) over the group
  prm.head_grp = head_group(static_cast<double>(std::max(Skv, 1)) * D * 2 * 2 * (tnd ? 1 : B) / prm.group, Nq);

  qbsa_status st;
  if ((st = make_map(&prm.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, qd, qs, 64)) != QBSA_OK) return st;
  if ((st = make_map(&prm.tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, kd, ks, 64)) != QBSA_OK) return st;
  if ((st = make_map(&prm.tm_v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, kd, ks, 64)) != QBSA_OK) return st;
  // atten_mask / pse tiles by TMA when their rows and bases are 16-byte aligned
  if (atten_mask && Skv % 16 == 0 && reinterpret_cast<uintptr_t>(atten_mask) % 16 == 0) {
    prm.mask_heads = mask_shape == QBSA_MASK_BNSS;
    prm.mask_batches = mask_shape != QBSA_MASK_SS;
    const uint64_t nh = prm.mask_heads ? Nq : 1, nb = prm.mask_batches ? B : 1;
    const uint64_t md[4] = {(uint64_t)Skv, (uint64_t)Sq, nh, nb};
    const uint64_t ms[3] = {(uint64_t)Skv, (uint64_t)Sq * Skv, nh * Sq * Skv};
    if ((st = make_map(&prm.tm_m, CU_TENSOR_MAP_DATA_TYPE_UINT8, atten_mask, md, ms, 128)) != QBSA_OK) return st;
    prm.mask_tma = 1;
  }
  if (pse && Skv % 8 == 0 && reinterpret_cast<uintptr_t>(pse) % 16 == 0) {
    prm.pse_batches = !pse_batch_bcast;
    const uint64_t nb = prm.pse_batches ? B : 1;
    const uint64_t pd[4] = {(uint64_t)Skv, (uint64_t)Sq, (uint64_t)Nq, nb};
    const uint64_t ps[3] = {2ull * Skv, 2ull * Sq * Skv, 2ull * Nq * Sq * Skv};
    if ((st = make_map(&prm.tm_p, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, pse, pd, ps, 64)) != QBSA_OK) return st;
    prm.pse_tma = 1;
  }

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // unmasked D = 128 BNSD / BSND (no atten_mask, pse or block mask; a band that covers
  // every (i, j)): two query tiles per CTA sharing each K/V tile
  const bool pair_path = D == 128 && !tnd && !atten_mask && !pse && !block_mask && sparse_mode == 0 &&
                         pre >= (int64_t)Sq - 1 && nxt >= (int64_t)Skv - 1;
  if (pair_path) {
    qbsa::PairParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.tm_q = prm.tm_q;
    pp.tm_k = prm.tm_k;
    pp.tm_v = prm.tm_v;
    if ((st = make_map(&pp.tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, attention_out, qd, qs, 64)) != QBSA_OK) return st;
    pp.softmax_max = softmax_max;
    pp.softmax_sum = softmax_sum;
    pp.B = B;
    pp.Nq = Nq;
    pp.Nkv = Nkv;
    pp.Sq = Sq;
    pp.Skv = Skv;
    pp.group = Nq / Nkv;
    pp.n_qtiles = (Sq + qbsa::kTile - 1) / qbsa::kTile;
    pp.n_ktiles = (Skv + qbsa::kTile - 1) / qbsa::kTile;
    pp.n_pair = (pp.n_qtiles + 1) / 2;
    pp.n_rank = B * pp.n_pair;
    pp.head_grp = prm.head_grp;
    pp.scale = scale;
    const int64_t n_pw = (int64_t)pp.n_rank * Nq;
    if ((st = set_smem(qbsa::attn_pair_kernel, qbsa::PairCfg::kSmemBytes)) != QBSA_OK) return st;
    qbsa::attn_pair_kernel<<<dim3(static_cast<unsigned>(n_pw)), qbsa::PairCfg::kThreads, qbsa::PairCfg::kSmemBytes,
                             s>>>(pp);
    return check_launch("attn_pair_kernel launch");
  }
  // D = 128 under band / causal masks or TND, without an explicit atten_mask, pse or block
  // mask: two query tiles per CTA with their own K-tile ranges
  const bool pair_masked_path = D == 128 && !atten_mask && !pse && !block_mask;
  if (pair_masked_path) {
    qbsa::PairMaskedParams pp;
    memset(&pp, 0, sizeof(pp));
    pp.tm_q = prm.tm_q;
    pp.tm_k = prm.tm_k;
    pp.tm_v = prm.tm_v;
    if (!tnd &&
        (st = make_map(&pp.tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, attention_out, qd, qs, 64)) != QBSA_OK)
      return st;
    pp.out = static_cast<__nv_bfloat16*>(attention_out);
    pp.softmax_max = softmax_max;
    pp.softmax_sum = softmax_sum;
    pp.o_row_stride = prm.o_row_stride;
    pp.o_head_stride = prm.o_head_stride;
    pp.stat_head_stride = prm.stat_head_stride;
    pp.stat_batch_stride = prm.stat_batch_stride;
    pp.pre_tokens = pre;
    pp.next_tokens = nxt;
    pp.B = B;
    pp.Nq = Nq;
    pp.Nkv = Nkv;
    pp.Sq = Sq;
    pp.Skv = Skv;
    pp.group = Nq / Nkv;
    pp.sparse_mode = sparse_mode;
    pp.tnd = tnd ? 1 : 0;
    pp.head_grp = prm.head_grp;
    pp.scale = scale;
    int64_t n_pairs = 0;
    if (tnd) {
      pp.n_seq = prm.n_seq;
      for (int i = 0; i < prm.n_seq; ++i) {
        pp.seq_q_start[i] = prm.seq_q_start[i];
        pp.seq_q_len[i] = prm.seq_q_len[i];
        pp.seq_kv_start[i] = prm.seq_kv_start[i];
        pp.seq_kv_len[i] = prm.seq_kv_len[i];
        pp.seq_pair_start[i] = static_cast<int>(n_pairs);
        n_pairs += ((prm.seq_q_len[i] + qbsa::kTile - 1) / qbsa::kTile + 1) / 2;
      }
      pp.seq_pair_start[prm.n_seq] = static_cast<int>(n_pairs);
    } else {
      pp.n_qtiles = (Sq + qbsa::kTile - 1) / qbsa::kTile;
      pp.n_pair = (pp.n_qtiles + 1) / 2;
      n_pairs = (int64_t)B * pp.n_pair;
    }
    pp.n_rank = static_cast<int>(n_pairs);
    const int64_t n_pw = n_pairs * Nq;
    if (n_pw == 0) return QBSA_OK;
    if ((st = set_smem(qbsa::attn_pair_masked_kernel, qbsa::PairCfg::kSmemBytes)) != QBSA_OK) return st;
    qbsa::attn_pair_masked_kernel<<<dim3(static_cast<unsigned>(n_pw)), qbsa::PairMaskedCfg::kThreads,
                                    qbsa::PairCfg::kSmemBytes, s>>>(pp);
    return check_launch("attn_pair_masked_kernel launch");
  }
  if (block_mask) {
    prm.block_mask = block_mask;
    prm.mask_nkb = (Skv + qbsa::kTile - 1) / qbsa::kTile;
  }
  return D == 128 ? launch_dense<128>(prm, n_work, s) : launch_dense<64>(prm, n_work, s);
}

qbsa_status attn_fwd(const void* q, const void* k, const void* v, int B, int Nq, int Nkv, int Sq, int Skv, int D,
                     int head_num, qbsa_layout input_layout, const uint8_t* atten_mask, qbsa_mask_shape mask_shape,
                     const void* pse, int pse_batch_bcast, float scale, float keep_prob, int sparse_mode,
                     int64_t pre_tokens, int64_t next_tokens, const int64_t* actual_seq_qlen,
                     const int64_t* actual_seq_kvlen, void* attention_out, float* softmax_max, float* softmax_sum,
                     void* stream) {
  return attn_fwd_impl(q, k, v, B, Nq, Nkv, Sq, Skv, D, head_num, input_layout, atten_mask, mask_shape, pse,
                       pse_batch_bcast, scale, keep_prob, sparse_mode, pre_tokens, next_tokens, actual_seq_qlen,
                       actual_seq_kvlen, attention_out, softmax_max, softmax_sum, stream, nullptr);
}

qbsa_status bsa_fwd(const void* q, const void* k, const void* v, const uint8_t* block_mask, int B, int Nq, int Nkv,
                    int Sq, int Skv, int D, float scale, void* attention_out, float* softmax_max, float* softmax_sum,
                    void* stream) {
  if (!block_mask) return fail(QBSA_ERR_INVALID, "bsa_fwd needs a block_mask");
  if ((Skv + qbsa::kTile - 1) / qbsa::kTile > qbsa::DenseCfg<128>::kMaxListed)
    return fail(QBSA_ERR_UNSUPPORTED, "ceil(Skv/128) exceeds %d", qbsa::DenseCfg<128>::kMaxListed);
  return attn_fwd_impl(q, k, v, B, Nq, Nkv, Sq, Skv, D, Nq, QBSA_LAYOUT_BNSD, nullptr, QBSA_MASK_NONE, nullptr, 0,
                       scale, 1.0f, 0, INT64_C(2147483647), INT64_C(2147483647), nullptr, nullptr, attention_out,
                       softmax_max, softmax_sum, stream, block_mask);
}

// ------------------------------------------------------------------------------
// qbsa_fwd
// ------------------------------------------------------------------------------

}  // extern "C"

// The shape checks qbsa_fwd and qbsa_fwd_host share.
static qbsa_status qbsa_shape_check(int B, int Nq, int Nkv, int Sq, int Skv, int D, float scale) {
  if (B < 1 || Nq < 1 || Nkv < 1 || Sq < 0 || Skv < 0) return fail(QBSA_ERR_INVALID, "B, Nq, Nkv >= 1 and Sq, Skv >= 0");
  if (Nq % Nkv != 0) return fail(QBSA_ERR_INVALID, "Nq (%d) must be a multiple of Nkv (%d)", Nq, Nkv);
  if (D != 128) return fail(QBSA_ERR_UNSUPPORTED, "qbsa_fwd supports D = 128 (got %d)", D);
  if (!std::isfinite(scale)) return fail(QBSA_ERR_INVALID, "scale must be finite");
  if (Sq > kMaxLen || Skv > kMaxLen) return fail(QBSA_ERR_UNSUPPORTED, "sequence length above %lld", (long long)kMaxLen);
  const int nkb = (Skv + 127) / 128;
  if (nkb > qbsa::kQbsaMaxKBlocks)
    return fail(QBSA_ERR_UNSUPPORTED, "ceil(Skv/128) = %d exceeds %d", nkb, qbsa::kQbsaMaxKBlocks);
  return QBSA_OK;
}

extern "C" {

qbsa_status qbsa_fwd(const int8_t* q_i8, const int8_t* k_i8, const float* q_block_scale, const float* k_block_scale,
                     const uint8_t* v_fp8, const float* v_channel_scale, const uint8_t* block_mask, int B, int Nq,
                     int Nkv, int Sq, int Skv, int D, float scale, void* attention_out, float* softmax_max,
                     float* softmax_sum, void* stream) {
  if (!q_i8 || !k_i8 || !q_block_scale || !k_block_scale || !v_fp8 || !v_channel_scale || !block_mask ||
      !attention_out)
    return fail(QBSA_ERR_INVALID, "all tensor arguments except the softmax statistics must be non-null");
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v_fp8) || !aligned16(attention_out))
    return fail(QBSA_ERR_INVALID, "q_i8, k_i8, v_fp8 and attention_out must be 16-byte aligned");
  {
    const qbsa_status sc = qbsa_shape_check(B, Nq, Nkv, Sq, Skv, D, scale);
    if (sc != QBSA_OK) return sc;
  }
  const int nqb = (Sq + 127) / 128, nkb = (Skv + 127) / 128;
  if (Sq == 0) return QBSA_OK;

  qbsa::QbsaParams prm;
  memset(&prm, 0, sizeof(prm));
  prm.q_scale = q_block_scale;
  prm.k_scale = k_block_scale;
  prm.v_scale = v_channel_scale;
  prm.block_mask = block_mask;
  prm.out = static_cast<__nv_bfloat16*>(attention_out);
  prm.softmax_max = softmax_max;
  prm.softmax_sum = softmax_sum;
  prm.B = B;
  prm.Nq = Nq;
  prm.Nkv = Nkv;
  prm.Sq = Sq;
  prm.Skv = Skv;
  prm.group = Nq / Nkv;
  prm.nqb = nqb;
  prm.nkb = nkb;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.n_pair = (nqb + 1) / 2;
  prm.n_rank = B * prm.n_pair;
  // K8 + V8 bytes of one query head: one kv head over all batches, shared by the group
  prm.head_grp = head_group(static_cast<double>(std::max(Skv, 1)) * 128 * 2 * B / prm.group, Nq);
  const int64_t n_work = (int64_t)B * prm.n_pair * Nq;
  if (n_work > 0x7fffffffLL) return fail(QBSA_ERR_UNSUPPORTED, "too many query blocks");
  if (Skv == 0) {
    // no key: every row is fully masked; keep the kernel path (no block is visited)
  }
  const uint64_t qd[4] = {128, (uint64_t)Sq, (uint64_t)Nq, (uint64_t)B};
  const uint64_t kd[4] = {128, (uint64_t)std::max(Skv, 1), (uint64_t)Nkv, (uint64_t)B};
  const uint64_t qs[3] = {128, (uint64_t)Sq * 128, (uint64_t)Nq * Sq * 128};
  const uint64_t ks[3] = {128, (uint64_t)std::max(Skv, 1) * 128, (uint64_t)Nkv * std::max(Skv, 1) * 128};
  qbsa_status st;
  if ((st = make_map(&prm.tm_q, CU_TENSOR_MAP_DATA_TYPE_UINT8, q_i8, qd, qs, 128)) != QBSA_OK) return st;
  if ((st = make_map(&prm.tm_k, CU_TENSOR_MAP_DATA_TYPE_UINT8, k_i8, kd, ks, 128)) != QBSA_OK) return st;
  if ((st = make_map(&prm.tm_v, CU_TENSOR_MAP_DATA_TYPE_UINT8, v_fp8, kd, ks, 128)) != QBSA_OK) return st;
  const uint64_t os[3] = {256, (uint64_t)Sq * 256, (uint64_t)Nq * Sq * 256};
  if ((st = make_map(&prm.tm_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, attention_out, qd, os, 64)) != QBSA_OK) return st;
  prm.mask_v16 = (nkb % 16 == 0) && aligned16(block_mask);
  if ((st = set_smem(qbsa::attn_qbsa_kernel, qbsa::QbsaCfg::kSmemBytes)) != QBSA_OK) return st;
  qbsa::attn_qbsa_kernel<<<dim3(static_cast<unsigned>(n_work)), qbsa::QbsaCfg::kThreads, qbsa::QbsaCfg::kSmemBytes,
                           static_cast<cudaStream_t>(stream)>>>(prm);
  return check_launch("attn_qbsa_kernel launch");
}

// ------------------------------------------------------------------------------
// quantisers
// ------------------------------------------------------------------------------

qbsa_status qbsa_quantize_qk(const void* x_bf16, int B, int N, int S, int D, int8_t* codes, float* scales,
                             void* stream) {
  if (!x_bf16 || !codes || !scales) return fail(QBSA_ERR_INVALID, "null pointer");
  if (B < 1 || N < 1 || S < 1 || D < 1) return fail(QBSA_ERR_INVALID, "B, N, S, D must be >= 1");
  if (D != 64 && D != 128 && D != 256) return fail(QBSA_ERR_UNSUPPORTED, "D must be 64, 128 or 256 (got %d)", D);
  if (!aligned16(x_bf16) || !aligned16(codes)) return fail(QBSA_ERR_INVALID, "x and codes must be 16-byte aligned");
  if (S > kMaxLen) return fail(QBSA_ERR_UNSUPPORTED, "sequence length above %lld", (long long)kMaxLen);
  const int nblk = (S + 127) / 128;
  if (N > 65535 || B > 65535) return fail(QBSA_ERR_UNSUPPORTED, "grid too large");
  const dim3 grid(nblk, N, B);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(x_bf16);
  if (D == 64) qbsa::quantize_qk_kernel<64><<<grid, qbsa::kQuantThreads, 0, st>>>(x, N, S, codes, scales);
  else if (D == 128) qbsa::quantize_qk_kernel<128><<<grid, qbsa::kQuantThreads, 0, st>>>(x, N, S, codes, scales);
  else qbsa::quantize_qk_kernel<256><<<grid, qbsa::kQuantThreads, 0, st>>>(x, N, S, codes, scales);
  return check_launch("quantize_qk_kernel launch");
}

}  // extern "C"

namespace {

// Scratch of the V quantiser: the per-head column maxima (float bits), zeroed before the first pass.
int64_t v_quant_scratch_words(int64_t H, int D) { return H * D; }

// Validates the V quantiser's arguments; on success fills the launch parameters (scratch
// pointer excluded).
qbsa_status v_quant_setup(const void* v_bf16, int B, int N, int S, int D, uint8_t* codes, float* scales,
                          qbsa::VQuantParams* prm) {
  if (!v_bf16 || !codes || !scales) return fail(QBSA_ERR_INVALID, "null pointer");
  if (B < 1 || N < 1 || S < 1 || D < 1) return fail(QBSA_ERR_INVALID, "B, N, S, D must be >= 1");
  if (D != 64 && D != 128 && D != 256) return fail(QBSA_ERR_UNSUPPORTED, "D must be 64, 128 or 256 (got %d)", D);
  if (!aligned16(v_bf16) || !aligned16(codes) || !aligned16(scales))
    return fail(QBSA_ERR_INVALID, "v, codes and scales must be 16-byte aligned");
  if (S > kMaxLen) return fail(QBSA_ERR_UNSUPPORTED, "sequence length above %lld", (long long)kMaxLen);
  const int rows = D == 64 ? qbsa::VQuantCfg<64>::kRows : D == 128 ? qbsa::VQuantCfg<128>::kRows
                                                                   : qbsa::VQuantCfg<256>::kRows;
  const int64_t H = (int64_t)B * N;
  const int64_t n_ch = (S + rows - 1) / rows;
  if (H * n_ch > 0x7fffffffLL) return fail(QBSA_ERR_UNSUPPORTED, "too many (head, chunk) blocks");
  memset(prm, 0, sizeof(*prm));
  prm->v = static_cast<const __nv_bfloat16*>(v_bf16);
  prm->codes = codes;
  prm->scales = scales;
  prm->H = static_cast<int>(H);
  prm->S = S;
  prm->n_ch = static_cast<int>(n_ch);
  return QBSA_OK;
}

// Both passes, queued on `st` (prm.amax must already be zeroed on `st`).
qbsa_status v_quant_launch(const qbsa::VQuantParams& prm, int D, cudaStream_t st) {
  const unsigned grid = static_cast<unsigned>((int64_t)prm.H * prm.n_ch);
  if (D == 64) qbsa::v_colmax_kernel<64><<<grid, qbsa::kQuantThreads, 0, st>>>(prm);
  else if (D == 128) qbsa::v_colmax_kernel<128><<<grid, qbsa::kQuantThreads, 0, st>>>(prm);
  else qbsa::v_colmax_kernel<256><<<grid, qbsa::kQuantThreads, 0, st>>>(prm);
  qbsa_status r = check_launch("v_colmax_kernel launch");
  if (r != QBSA_OK) return r;
  if (D == 64) qbsa::v_quant_kernel<64><<<grid, qbsa::kQuantThreads, 0, st>>>(prm);
  else if (D == 128) qbsa::v_quant_kernel<128><<<grid, qbsa::kQuantThreads, 0, st>>>(prm);
  else qbsa::v_quant_kernel<256><<<grid, qbsa::kQuantThreads, 0, st>>>(prm);
  return check_launch("v_quant_kernel launch");
}

// Per device, a stream-ordered memory pool whose memory stays with the library between calls
// (release threshold: everything), so that scratch and staging buffers cost no fresh
// allocation after the first call of a size.  (The device's default pool returns its memory
// at every synchronisation, after which each allocation maps memory again on the host's
// issue path.)
constexpr int kPoolDevices = 64;
std::mutex g_pool_mu;
cudaMemPool_t g_pool[kPoolDevices] = {};

qbsa_status library_pool(cudaMemPool_t* out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kPoolDevices) return fail(QBSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_pool_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props;
    memset(&props, 0, sizeof(props));
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if ((e = cudaMemPoolCreate(&pool, &props)) != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
    uint64_t keep = ~0ull;
    if ((e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep)) != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return cuda_fail(e, "cudaMemPoolSetAttribute");
    }
    g_pool[dev] = pool;
  }
  *out = g_pool[dev];
  return QBSA_OK;
}

}  // namespace

extern "C" {

qbsa_status qbsa_quantize_v(const void* v_bf16, int B, int N, int S, int D, uint8_t* codes, float* scales,
                            void* stream) {
  qbsa::VQuantParams prm;
  qbsa_status st = v_quant_setup(v_bf16, B, N, S, D, codes, scales, &prm);
  if (st != QBSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(v_quant_scratch_words(prm.H, D)) * sizeof(unsigned int);
  cudaMemPool_t pool = nullptr;
  if ((st = library_pool(&pool)) != QBSA_OK) return st;
  void* scratch = nullptr;
  cudaError_t e = cudaMallocFromPoolAsync(&scratch, bytes, pool, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync (V quantiser scratch)");
  e = cudaMemsetAsync(scratch, 0, bytes, s);
  if (e != cudaSuccess) {
    cudaFreeAsync(scratch, s);
    return cuda_fail(e, "cudaMemsetAsync (V quantiser scratch)");
  }
  prm.amax = static_cast<unsigned int*>(scratch);
  st = v_quant_launch(prm, D, s);
  e = cudaFreeAsync(scratch, s);
  if (st != QBSA_OK) return st;
  if (e != cudaSuccess) return cuda_fail(e, "cudaFreeAsync (V quantiser scratch)");
  return QBSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------
// V quantiser with a library-resident scratch array (no allocation per call)
// ------------------------------------------------------------------------------
//
// Some callers cannot allocate device memory at the moment they quantise V: code that
// runs inside a custom allocator or a memory-pool callback, callers whose device heap is
// fully reserved up front (a serving process that pre-plans every byte), or runtimes
// that forbid cudaMalloc / cudaMallocAsync on their streams.  This entry point gives them
// the same V quantiser with its scratch (the per-head column maxima) in a fixed array that
// lives in the library's device image.

namespace {

constexpr int64_t kNoAllocScratchWords = 65536;  // 256 KiB per device, held until the process exits
__device__ __align__(256) unsigned int g_vq_scratch[kNoAllocScratchWords];

constexpr int kMaxDevices = 64;
std::mutex g_vq_scratch_mu;
unsigned int* g_vq_scratch_ptr[kMaxDevices] = {};

// Device address of g_vq_scratch on the current device, looked up once per device (in
// host code the symbol is only a host-side stand-in, never a device address).
qbsa_status vq_scratch_address(unsigned int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(QBSA_ERR_UNSUPPORTED, "device ordinal %d above %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_vq_scratch_mu);
  if (!g_vq_scratch_ptr[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_vq_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (V quantiser scratch)");
    g_vq_scratch_ptr[dev] = static_cast<unsigned int*>(ptr);
  }
  *out = g_vq_scratch_ptr[dev];
  return QBSA_OK;
}

}  // namespace

extern "C" {

qbsa_status qbsa_quantize_v_noalloc(const void* v_bf16, int B, int N, int S, int D, uint8_t* codes, float* scales,
                                    void* stream) {
  qbsa::VQuantParams prm;
  qbsa_status st = v_quant_setup(v_bf16, B, N, S, D, codes, scales, &prm);
  if (st != QBSA_OK) return st;
  const int64_t words = v_quant_scratch_words(prm.H, D);
  if (words > kNoAllocScratchWords)
    return fail(QBSA_ERR_UNSUPPORTED,
                "qbsa_quantize_v_noalloc: B*N*D = %lld scratch words exceed the fixed %lld (256 KiB); "
                "use qbsa_quantize_v", (long long)words, (long long)kNoAllocScratchWords);
  unsigned int* w = nullptr;
  if ((st = vq_scratch_address(&w)) != QBSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(w, 0, static_cast<size_t>(words) * sizeof(unsigned int), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (V quantiser scratch)");
  prm.amax = w;
  return v_quant_launch(prm, D, s);
}

}  // extern "C"

extern "C" {

// ------------------------------------------------------------------------------
// schedule export, mask compaction hook, error word
// ------------------------------------------------------------------------------

qbsa_status attn_tile_schedule(int64_t sq, int64_t skv, int sparse_mode, int64_t pre_tokens, int64_t next_tokens,
                               int32_t* kt_begin, int32_t* kt_end, int32_t* full_begin, int32_t* full_end,
                               int64_t n_qtiles) {
  if (!kt_begin || !kt_end || !full_begin || !full_end) return fail(QBSA_ERR_INVALID, "null output array");
  if (sq < 0 || skv < 0 || sq > kMaxLen || skv > kMaxLen) return fail(QBSA_ERR_INVALID, "bad sequence lengths");
  if (sparse_mode != 0 && sparse_mode != 2 && sparse_mode != 3)
    return fail(QBSA_ERR_UNSUPPORTED, "sparse_mode %d is not implemented", sparse_mode);
  if (n_qtiles != (sq + qbsa::kTile - 1) / qbsa::kTile) return fail(QBSA_ERR_INVALID, "n_qtiles must be ceil(sq/128)");
  const int64_t pre = std::max(-kTokenClamp, std::min(kTokenClamp, pre_tokens));
  const int64_t nxt = std::max(-kTokenClamp, std::min(kTokenClamp, next_tokens));
  const qbsa::Band band = qbsa::band_of(sparse_mode, pre, nxt, sq, skv);
  for (int64_t t = 0; t < n_qtiles; ++t) {
    const qbsa::TileRange r = qbsa::tile_range((int)t, sq, skv, band);
    kt_begin[t] = r.kt_begin;
    kt_end[t] = r.kt_end;
    full_begin[t] = r.full_begin;
    full_end[t] = r.full_end;
  }
  return QBSA_OK;
}

qbsa_status qbsa_block_lists(const uint8_t* block_mask, int64_t rows, int n_kb, int32_t* lists, int32_t* counts,
                             void* stream) {
  if (!block_mask || !lists || !counts) return fail(QBSA_ERR_INVALID, "null pointer");
  if (rows < 0 || n_kb < 1 || n_kb > qbsa::kQbsaMaxKBlocks) return fail(QBSA_ERR_INVALID, "bad rows / n_kb");
  if (rows == 0) return QBSA_OK;
  const int64_t grid = (rows + 3) / 4;
  if (grid > 0x7fffffffLL) return fail(QBSA_ERR_UNSUPPORTED, "too many rows");
  qbsa::qbsa_block_lists_kernel<<<(unsigned)grid, 128, 0, static_cast<cudaStream_t>(stream)>>>(
      block_mask, (int)rows, n_kb, lists, counts);
  return check_launch("qbsa_block_lists_kernel launch");
}

// ------------------------------------------------------------------------------
// block-mask estimation
// ------------------------------------------------------------------------------

qbsa_status qbsa_block_mean(const void* x, int B, int N, int S, int D, float* x_mean, void* stream) {
  if (!x || !x_mean) return fail(QBSA_ERR_INVALID, "x and x_mean must be non-null");
  if (!aligned16(x)) return fail(QBSA_ERR_INVALID, "x must be 16-byte aligned");
  if (B < 1 || N < 1 || S < 1) return fail(QBSA_ERR_INVALID, "B, N, S >= 1");
  if (D != 64 && D != 128 && D != 256) return fail(QBSA_ERR_UNSUPPORTED, "block mean supports D in {64,128,256}");
  if (S > kMaxLen) return fail(QBSA_ERR_UNSUPPORTED, "sequence length above %lld", (long long)kMaxLen);
  const int nb = (S + qbsa::kTile - 1) / qbsa::kTile;
  const int64_t n_cta = (int64_t)B * N * nb;
  if (n_cta > 0x7fffffffLL) return fail(QBSA_ERR_UNSUPPORTED, "too many blocks");
  qbsa::block_mean_kernel<<<dim3(static_cast<unsigned>(n_cta)), qbsa::kEstThreads, 0,
                            static_cast<cudaStream_t>(stream)>>>(static_cast<const __nv_bfloat16*>(x), S, D, nb,
                                                                  x_mean);
  return check_launch("block_mean_kernel launch");
}

qbsa_status qbsa_block_topk(const float* q_mean, const float* k_mean, int B, int Nq, int Nkv, int nqb, int nkb, int D,
                            float scale, int n_keep, uint8_t* block_mask, float* block_scores, void* stream) {
  if (!q_mean || !k_mean || !block_mask) return fail(QBSA_ERR_INVALID, "q_mean, k_mean and block_mask must be non-null");
  if (B < 1 || Nq < 1 || Nkv < 1 || nqb < 1 || nkb < 1 || D < 1) return fail(QBSA_ERR_INVALID, "sizes must be >= 1");
  if (Nq % Nkv != 0) return fail(QBSA_ERR_INVALID, "Nq (%d) must be a multiple of Nkv (%d)", Nq, Nkv);
  if (nkb > qbsa::kTopkMaxKBlocks) return fail(QBSA_ERR_UNSUPPORTED, "nkb above %d", qbsa::kTopkMaxKBlocks);
  if (D > 1024 || D % 4 != 0) return fail(QBSA_ERR_UNSUPPORTED, "D must be a multiple of 4, at most 1024");
  if (!aligned16(k_mean)) return fail(QBSA_ERR_INVALID, "k_mean must be 16-byte aligned");
  if (n_keep < 1 || n_keep > nkb) return fail(QBSA_ERR_INVALID, "n_keep must be in [1, nkb]");
  if (!std::isfinite(scale)) return fail(QBSA_ERR_INVALID, "scale must be finite");
  const int64_t n_cta = (int64_t)B * Nq * ((nqb + qbsa::kTopkGroup - 1) / qbsa::kTopkGroup);
  if (n_cta > 0x7fffffffLL) return fail(QBSA_ERR_UNSUPPORTED, "too many query blocks");
  const int smem = qbsa::topk_smem_bytes(nkb, D);
  qbsa_status st;
  if ((st = set_smem(qbsa::block_topk_kernel, smem)) != QBSA_OK) return st;
  qbsa::block_topk_kernel<<<dim3(static_cast<unsigned>(n_cta)), qbsa::kTopkThreads, smem,
                            static_cast<cudaStream_t>(stream)>>>(q_mean, k_mean, Nq, Nq / Nkv, nqb, nkb, D, scale,
                                                                  n_keep, block_mask, block_scores);
  return check_launch("block_topk_kernel launch");
}

qbsa_status qbsa_block_topk_keep(const float* q_mean, const float* k_mean, int B, int Nq, int Nkv, int nqb, int nkb,
                                 int D, float scale, double keep, uint8_t* block_mask, float* block_scores,
                                 int* n_keep_out, void* stream) {
  if (!(keep >= 0.0 && keep <= 1.0)) return fail(QBSA_ERR_INVALID, "keep must be in [0, 1]");
  if (nkb < 1) return fail(QBSA_ERR_INVALID, "sizes must be >= 1");
  // blocks kept per query block: keep * nkb rounded to nearest (ties to even), at least 1
  const int n_keep = std::max(1, std::min(nkb, static_cast<int>(std::nearbyint(keep * nkb))));
  if (n_keep_out) *n_keep_out = n_keep;
  return qbsa_block_topk(q_mean, k_mean, B, Nq, Nkv, nqb, nkb, D, scale, n_keep, block_mask, block_scores, stream);
}

namespace qbsa {
// Failure-detection self-test: one thread waits, through the kernels' own bounded wait, on
// an mbarrier phase that nothing completes; the wait gives up after its time limit, records
// the timeout in the device error word and the kernel returns normally.
__global__ void wait_selftest_kernel() {
  __shared__ uint64_t barrier;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  const uint32_t bar = smem_u32(&barrier);
  mbar_init(bar, 1);
  fence_mbar_init();
  mbar_wait(bar, 0, &abort_flag);  // no arrival ever comes
}
}  // namespace qbsa

qbsa_status qbsa_wait_selftest(void* stream) {
  qbsa::wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return check_launch("wait_selftest_kernel launch");
}

qbsa_status qbsa_check(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned int word = 0;
  e = cudaMemcpyFromSymbol(&word, qbsa::g_device_error, sizeof(word));
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (word != 0) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(qbsa::g_device_error, &zero, sizeof(zero));
    return fail(QBSA_ERR_TIMEOUT, "a kernel wait exceeded its time limit (device error word %u)", word);
  }
  return QBSA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------------------
// qbsa_fwd on host buffers: chunked copies that overlap the kernel
// ------------------------------------------------------------------------------
//
// Per device the library keeps two non-blocking copy streams (host -> device, device ->
// host); the call's device buffers come from the library's memory pool (above), so they cost
// no fresh allocation after the first call of that size.

namespace {

struct HostPathState {
  bool ready = false;
  cudaStream_t s_in = nullptr;
  cudaStream_t s_out = nullptr;
  cudaMemPool_t pool = nullptr;
};

constexpr int kHostPathDevices = 64;
std::mutex g_host_path_mu;
HostPathState g_host_path[kHostPathDevices];

qbsa_status host_path_state(HostPathState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kHostPathDevices) return fail(QBSA_ERR_UNSUPPORTED, "device ordinal %d", dev);
  std::lock_guard<std::mutex> lock(g_host_path_mu);
  HostPathState& st = g_host_path[dev];
  if (!st.ready) {
    if ((e = cudaStreamCreateWithFlags(&st.s_in, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamCreateWithFlags (copy-in stream)");
    if ((e = cudaStreamCreateWithFlags(&st.s_out, cudaStreamNonBlocking)) != cudaSuccess)
      return cuda_fail(e, "cudaStreamCreateWithFlags (copy-out stream)");
    const qbsa_status ps = library_pool(&st.pool);
    if (ps != QBSA_OK) return ps;
    st.ready = true;
  }
  *out = &st;
  return QBSA_OK;
}

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

extern "C" {

qbsa_status qbsa_fwd_host(const int8_t* q_i8, const int8_t* k_i8, const float* q_block_scale,
                          const float* k_block_scale, const uint8_t* v_fp8, const float* v_channel_scale,
                          const uint8_t* block_mask, int B, int Nq, int Nkv, int Sq, int Skv, int D, float scale,
                          void* attention_out, float* softmax_max, float* softmax_sum, int n_chunks, void* stream) {
  if (!q_i8 || !k_i8 || !q_block_scale || !k_block_scale || !v_fp8 || !v_channel_scale || !block_mask ||
      !attention_out)
    return fail(QBSA_ERR_INVALID, "all tensor arguments except the softmax statistics must be non-null");
  if (n_chunks < 1) return fail(QBSA_ERR_INVALID, "n_chunks must be >= 1 (got %d)", n_chunks);
  {
    const qbsa_status sc = qbsa_shape_check(B, Nq, Nkv, Sq, Skv, D, scale);
    if (sc != QBSA_OK) return sc;
  }
  if (Sq == 0) return QBSA_OK;
  HostPathState* hp = nullptr;
  qbsa_status st = host_path_state(&hp);
  if (st != QBSA_OK) return st;

  const int group = Nq / Nkv;
  const int nqb = (Sq + 127) / 128, nkb = (Skv + 127) / 128;
  const size_t sq = static_cast<size_t>(Sq), skv = static_cast<size_t>(Skv), dd = static_cast<size_t>(D);
  // per-head sizes in bytes of every tensor; the device copies keep the host layout
  const size_t q_h = sq * dd, k_h = skv * dd, qs_h = nqb * 4ull, ks_h = nkb * 4ull, vs_h = dd * 4,
               m_h = static_cast<size_t>(nqb) * nkb, o_h = sq * dd * 2, st_h = sq * 4;
  const size_t nq = static_cast<size_t>(B) * Nq, nk = static_cast<size_t>(B) * Nkv;
  const size_t off_q = 0, off_k = off_q + round256(nq * q_h), off_v = off_k + round256(nk * k_h),
               off_qs = off_v + round256(nk * k_h), off_ks = off_qs + round256(nq * qs_h),
               off_vs = off_ks + round256(nk * ks_h), off_m = off_vs + round256(nk * vs_h),
               off_o = off_m + round256(nq * m_h), off_mx = off_o + round256(nq * o_h),
               off_sm = off_mx + round256(softmax_max ? nq * st_h : 0),
               total = off_sm + round256(softmax_sum ? nq * st_h : 0);

  cudaStream_t sc = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev_ready = nullptr, ev_in = nullptr, ev_comp = nullptr, ev_done = nullptr;
  uint8_t* dbuf = nullptr;
  cudaError_t e = cudaSuccess;
  const char* what = nullptr;
  auto ok = [&](cudaError_t r, const char* w) {
    if (r != cudaSuccess && e == cudaSuccess) {
      e = r;
      what = w;
    }
    return e == cudaSuccess;
  };
  if (ok(cudaEventCreateWithFlags(&ev_ready, cudaEventDisableTiming), "cudaEventCreate") &&
      ok(cudaEventCreateWithFlags(&ev_in, cudaEventDisableTiming), "cudaEventCreate") &&
      ok(cudaEventCreateWithFlags(&ev_comp, cudaEventDisableTiming), "cudaEventCreate") &&
      ok(cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming), "cudaEventCreate") &&
      ok(cudaMallocFromPoolAsync(reinterpret_cast<void**>(&dbuf), total, hp->pool, sc), "cudaMallocFromPoolAsync") &&
      ok(cudaEventRecord(ev_ready, sc), "cudaEventRecord") &&
      ok(cudaStreamWaitEvent(hp->s_in, ev_ready, 0), "cudaStreamWaitEvent")) {
    // chunks: whole GQA groups of kv heads [g0, g1) of one batch entry
    const int per_b = std::max(1, std::min(Nkv, (n_chunks + B - 1) / B));
    const auto h2d = [&](size_t off, const void* host, size_t bytes) {
      return ok(cudaMemcpyAsync(dbuf + off, host, bytes, cudaMemcpyHostToDevice, hp->s_in), "cudaMemcpyAsync (in)");
    };
    const auto d2h = [&](void* host, size_t off, size_t bytes) {
      return ok(cudaMemcpyAsync(host, dbuf + off, bytes, cudaMemcpyDeviceToHost, hp->s_out), "cudaMemcpyAsync (out)");
    };
    for (int b = 0; b < B && e == cudaSuccess && st == QBSA_OK; ++b) {
      for (int c = 0; c < per_b && e == cudaSuccess && st == QBSA_OK; ++c) {
        const int g0 = static_cast<int>((int64_t)c * Nkv / per_b), g1 = static_cast<int>((int64_t)(c + 1) * Nkv / per_b);
        if (g1 <= g0) continue;
        const size_t hq0 = static_cast<size_t>(b) * Nq + static_cast<size_t>(g0) * group;  // first query head
        const size_t hk0 = static_cast<size_t>(b) * Nkv + g0;                               // first kv head
        const size_t nhq = static_cast<size_t>(g1 - g0) * group, nhk = static_cast<size_t>(g1 - g0);
        const uint8_t* hq = reinterpret_cast<const uint8_t*>(q_i8);
        const uint8_t* hk = reinterpret_cast<const uint8_t*>(k_i8);
        const uint8_t* hqs = reinterpret_cast<const uint8_t*>(q_block_scale);
        const uint8_t* hks = reinterpret_cast<const uint8_t*>(k_block_scale);
        const uint8_t* hvs = reinterpret_cast<const uint8_t*>(v_channel_scale);
        if (!(h2d(off_q + hq0 * q_h, hq + hq0 * q_h, nhq * q_h) && h2d(off_k + hk0 * k_h, hk + hk0 * k_h, nhk * k_h) &&
              h2d(off_v + hk0 * k_h, v_fp8 + hk0 * k_h, nhk * k_h) &&
              h2d(off_qs + hq0 * qs_h, hqs + hq0 * qs_h, nhq * qs_h) &&
              h2d(off_ks + hk0 * ks_h, hks + hk0 * ks_h, nhk * ks_h) &&
              h2d(off_vs + hk0 * vs_h, hvs + hk0 * vs_h, nhk * vs_h) &&
              h2d(off_m + hq0 * m_h, block_mask + hq0 * m_h, nhq * m_h) &&
              ok(cudaEventRecord(ev_in, hp->s_in), "cudaEventRecord") &&
              ok(cudaStreamWaitEvent(sc, ev_in, 0), "cudaStreamWaitEvent")))
          break;
        st = qbsa_fwd(reinterpret_cast<const int8_t*>(dbuf + off_q + hq0 * q_h),
                      reinterpret_cast<const int8_t*>(dbuf + off_k + hk0 * k_h),
                      reinterpret_cast<const float*>(dbuf + off_qs + hq0 * qs_h),
                      reinterpret_cast<const float*>(dbuf + off_ks + hk0 * ks_h), dbuf + off_v + hk0 * k_h,
                      reinterpret_cast<const float*>(dbuf + off_vs + hk0 * vs_h), dbuf + off_m + hq0 * m_h, 1,
                      static_cast<int>(nhq), static_cast<int>(nhk), Sq, Skv, D, scale, dbuf + off_o + hq0 * o_h,
                      softmax_max ? reinterpret_cast<float*>(dbuf + off_mx + hq0 * st_h) : nullptr,
                      softmax_sum ? reinterpret_cast<float*>(dbuf + off_sm + hq0 * st_h) : nullptr, stream);
        if (st != QBSA_OK) break;
        if (!(ok(cudaEventRecord(ev_comp, sc), "cudaEventRecord") &&
              ok(cudaStreamWaitEvent(hp->s_out, ev_comp, 0), "cudaStreamWaitEvent") &&
              d2h(static_cast<uint8_t*>(attention_out) + hq0 * o_h, off_o + hq0 * o_h, nhq * o_h) &&
              (!softmax_max ||
               d2h(reinterpret_cast<uint8_t*>(softmax_max) + hq0 * st_h, off_mx + hq0 * st_h, nhq * st_h)) &&
              (!softmax_sum ||
               d2h(reinterpret_cast<uint8_t*>(softmax_sum) + hq0 * st_h, off_sm + hq0 * st_h, nhq * st_h))))
          break;
      }
    }
    // the buffers go back to the pool once the last copy out has read them
    ok(cudaEventRecord(ev_done, hp->s_out), "cudaEventRecord");
    ok(cudaStreamWaitEvent(sc, ev_done, 0), "cudaStreamWaitEvent");
  }
  if (dbuf) {
    const cudaError_t r = cudaFreeAsync(dbuf, sc);
    ok(r, "cudaFreeAsync");
  }
  ok(cudaStreamSynchronize(sc), "cudaStreamSynchronize");
  for (cudaEvent_t ev : {ev_ready, ev_in, ev_comp, ev_done})
    if (ev) cudaEventDestroy(ev);
  if (st != QBSA_OK) return st;
  if (e != cudaSuccess) return cuda_fail(e, what ? what : "qbsa_fwd_host");
  return QBSA_OK;
}

}  // extern "C"
