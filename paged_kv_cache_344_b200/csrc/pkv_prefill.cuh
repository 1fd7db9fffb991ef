// Multi-query attention over the paged cache (prefill / chunked append) on the
// 5th-generation tensor cores (sm_100a tcgen05, accumulators in TMEM).
//
// Sequence b holds L cached tokens whose last Q are this call's queries (their
// K/V already written by paged_kv_write).  Query i sits at position L - Q + i
// and attends causally to tokens 0 .. L - Q + i.  Each query row is the decode's
// softmax attention over its visible prefix ("PagedAttention: paging the KV
// cache like an OS pages memory", How it works: standard causal attention, only
// the storage layout changes).
//
// With Q > 1 this is a dense contraction, so it runs as tcgen05 MMAs:
//  * one CTA per (KV head, query tile, sequence); a query tile is 128 rows =
//    128/G query tokens x the G query heads of the KV head (rows ordered token,
//    head), loaded once by TMA into a 128-byte-swizzled K-major operand;
//  * K/V tiles of 64 tokens arrive by TMA as four 16-token boxes, each from the
//    physical block the table gives, double-buffered;
//  * S = Q K^T: M=128, N=64, K=16 per instruction, fp32 accumulator in TMEM;
//    each of the 4 warps reads its 32 rows of S (tcgen05.ld), masks causally,
//    and runs the online softmax (exp2, scale in log2 units) in registers;
//  * P (bf16) goes to shared memory in the swizzled K-major layout (into the K
//    tile it replaces); O += P V: M=128, N=D, K=16, V as an MN-major operand,
//    O accumulated in TMEM and rescaled in place when the running max grows;
//  * the epilogue reads O, divides by the row sums and writes bf16 rows.
// One elected thread issues every MMA; tcgen05.commit arrives on an mbarrier
// that the warps wait on (bounded).  TMEM is freed on every path.
#pragma once

#include "pkv_decode.cuh"

namespace pkv {

constexpr int kPrefillRows = 128;  // MMA M: query rows per CTA
constexpr int kPrefillKv = 64;     // MMA N of S: tokens per K/V tile

struct PrefillParams {
  void* out;                  // [T][Hq][D]
  const int32_t* block_tables;
  const int32_t* seq_lens;    // [B] cached tokens (queries included)
  const int32_t* cu_q;        // [B + 1] query row offsets
  int max_blocks;
  int max_seq_len;
  int Hq;
  int Hkv;
  int G;
  int TQ;                     // query tokens per tile = 128 / G
  int bs;
  int num_blocks;
  float scale_log2;
};

template <int D>
struct PrefillSmem {
  static constexpr int SUB = D / 64;                        // 128-byte column chunks
  static constexpr int kQBytes = SUB * kPrefillRows * 128;  // query tile
  static constexpr int kKvTile = SUB * kPrefillKv * 128;    // one of K or V
  static constexpr int kStage = 2 * kKvTile;
  // P (128 rows x 64 bf16) overwrites the K tile it was scored against when that
  // tile is large enough; otherwise it has a buffer of its own.
  static constexpr bool kPInK = kKvTile >= kPrefillRows * 128;
  static constexpr int kPBytes = kPInK ? 0 : kPrefillRows * 128;
  static constexpr int kOffQ = 0;
  static constexpr int kOffStage = kQBytes;
  static constexpr int kOffP = kOffStage + 2 * kStage;
  static constexpr int kOffBar = kOffP + kPBytes;
  static constexpr size_t kBytes = 1024 + (size_t)kOffBar + 8 * 8;
  // TMEM: S in columns [0, 64), O in [kOCol, kOCol + D).
  static constexpr uint32_t kOCol = D <= 64 ? 64 : (uint32_t)D;
  static constexpr uint32_t kCols = D <= 64 ? 128 : 2 * (uint32_t)D;
};

template <int D>
__device__ __forceinline__ void prefill_issue_kv(const PrefillParams& p, uint8_t* stage,
                                                 const CUtensorMap* tmK, const CUtensorMap* tmV,
                                                 uint64_t* bar, const int32_t* bt_row, int kvh,
                                                 int tile, int kv_end, uint64_t pol) {
  using S = PrefillSmem<D>;
  mbar_arrive_expect_tx(bar, S::kStage);
#pragma unroll
  for (int c = 0; c < kPrefillKv / kStageTokens; ++c) {
    const int t0 = tile * kPrefillKv + c * kStageTokens;
    int row = p.num_blocks * p.bs;  // past the end: the box is filled with zeros
    if (t0 < kv_end) {
      const int id = bt_row[t0 / p.bs];
      if (id >= 0 && id < p.num_blocks) row = id * p.bs + t0 % p.bs;
      else flag_error(PKV_DEVERR_BLOCK_ID);
    }
#pragma unroll
    for (int sb = 0; sb < S::SUB; ++sb) {
      tma_load_3d(stage + sb * (kPrefillKv * 128) + c * (kStageTokens * 128), tmK, bar, sb * 64,
                  kvh, row, pol);
      tma_load_3d(stage + S::kKvTile + sb * (kPrefillKv * 128) + c * (kStageTokens * 128), tmV,
                  bar, sb * 64, kvh, row, pol);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmQ,
                         const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV) {
  using S = PrefillSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  uint64_t* bar_kv = bar_q + 1;  // [2]
  uint64_t* bar_s = bar_q + 3;
  uint64_t* bar_o = bar_q + 4;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  if (*reinterpret_cast<volatile uint32_t*>(&g_device_errors) & PKV_DEVERR_TIMEOUT) return;
  const int kvh = blockIdx.x, qt = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G;
  const int q0 = p.cu_q[b];
  const int Q = p.cu_q[b + 1] - q0;
  const int i0 = qt * p.TQ;
  if (i0 >= Q) return;
  int L = p.seq_lens[b];
  const int Lcap = min(p.max_blocks * p.bs, p.max_seq_len);
  if (L > Lcap || Q > L) {
    if (threadIdx.x == 0 && qt == 0 && kvh == 0) flag_error(PKV_DEVERR_SEQLEN);
    if (Q > min(L, Lcap)) return;  // no consistent reading: rows are left unwritten
    L = Lcap;
  }
  const int ctx = L - Q;                      // cached tokens before the chunk
  const int i1 = min(Q, i0 + p.TQ);
  const int kv_end = ctx + i1;                // tokens any row of this tile sees
  const int n_kv = (kv_end + kPrefillKv - 1) / kPrefillKv;

  // Row of this thread: query token i, head g.  It sees tokens t < visible.
  const int r = threadIdx.x;
  const int i = i0 + r / G, g = r % G;
  const bool row_valid = i < Q;
  const int visible = min(ctx + i + 1, kv_end);

  if (warp == 0) {
    tmem_alloc(&s_tmem, S::kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(bar_q, 1);
    mbar_init(&bar_kv[0], 1);
    mbar_init(&bar_kv[1], 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    fence_mbar_init();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s_tmem;
  const uint32_t tmem_s = tmem;
  const uint32_t tmem_o = tmem + S::kOCol;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  const int32_t* bt_row = p.block_tables + (size_t)b * p.max_blocks;
  uint8_t* q_smem = smem + S::kOffQ;
  auto stage_ptr = [&](int st) { return smem + S::kOffStage + st * S::kStage; };
  const uint64_t pol = l2_policy_evict_first();
  if (threadIdx.x == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
    mbar_arrive_expect_tx(bar_q, S::kQBytes);
#pragma unroll
    for (int sb = 0; sb < S::SUB; ++sb)
      tma_load_3d(q_smem + sb * (kPrefillRows * 128), &tmQ, bar_q, sb * 64, kvh * G, q0 + i0, pol);
    prefill_issue_kv<D>(p, stage_ptr(0), &tmK, &tmV, &bar_kv[0], bt_row, kvh, 0, kv_end, pol);
    if (n_kv > 1)
      prefill_issue_kv<D>(p, stage_ptr(1), &tmK, &tmV, &bar_kv[1], bt_row, kvh, 1, kv_end, pol);
  }

  constexpr uint32_t kIdescS = umma_idesc_bf16(kPrefillRows, kPrefillKv, false);
  constexpr uint32_t kIdescO = umma_idesc_bf16(kPrefillRows, D, true);
  constexpr int KS = D / 16;
  const uint32_t q_addr = smem_u32(q_smem);
  float m_run = -INFINITY, l_run = 0.f;
  bool ok = true;

  for (int j = 0; j < n_kv; ++j) {
    const int st = j & 1;
    uint8_t* k_smem = stage_ptr(st);
    uint8_t* v_smem = k_smem + S::kKvTile;
    uint8_t* p_smem = S::kPInK ? k_smem : smem + S::kOffP;
    // S = Q K^T (one thread issues; the warps wait for the commit).
    if (threadIdx.x == 0) {
      bool ready = (j > 0) || mbar_wait_bounded(bar_q, 0);
      ready = ready && mbar_wait_bounded(&bar_kv[st], (uint32_t)((j >> 1) & 1));
      if (ready) {
        tc_fence_after_sync();
        const uint32_t k_addr = smem_u32(k_smem);
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          const uint64_t ad = umma_desc_sw128(q_addr + (kk / 4) * (kPrefillRows * 128) + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = umma_desc_sw128(k_addr + (kk / 4) * (kPrefillKv * 128) + (kk % 4) * 32, 16, 1024);
          umma_bf16(tmem_s, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
        }
        umma_commit(bar_s);
      }
    }
    ok = mbar_wait_bounded(bar_s, (uint32_t)(j & 1));
    if (__syncthreads_or(!ok)) break;
    tc_fence_after_sync();

    // Row softmax over this tile (the warp reads its 32 lanes of S).
    uint32_t sv[2][32];
    tmem_ld32(tmem_s + lane_base + 0, sv[0]);
    tmem_ld32(tmem_s + lane_base + 32, sv[1]);
    tmem_wait_ld();
    float x[kPrefillKv];
    float mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < kPrefillKv; ++c) {
      const int t = j * kPrefillKv + c;
      x[c] = t < visible ? __uint_as_float(sv[c / 32][c % 32]) * p.scale_log2 : -INFINITY;
      mx = fmaxf(mx, x[c]);
    }
    const float m_new = fmaxf(m_run, mx);
    const float alpha = exp2f(m_run - m_new);  // 0 for the first tile
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < kPrefillKv; ++c) {
      x[c] = exp2f(x[c] - m_new);
      sum += x[c];
    }
    l_run = l_run * alpha + sum;
    m_run = m_new;

    if (j > 0) {
      // The previous P V must be done before O is rescaled and P / stage st^1 reused.
      ok = mbar_wait_bounded(bar_o, (uint32_t)((j - 1) & 1));
      if (__syncthreads_or(!ok)) break;
      tc_fence_after_sync();
      if (threadIdx.x == 0 && j + 1 < n_kv)
        prefill_issue_kv<D>(p, stage_ptr(st ^ 1), &tmK, &tmV, &bar_kv[st ^ 1], bt_row, kvh, j + 1,
                            kv_end, pol);
      if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t ov[32];
          tmem_ld32(tmem_o + lane_base + cc * 32, ov);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          tmem_st32(tmem_o + lane_base + cc * 32, ov);
        }
        tmem_wait_st();
      }
    }

    // P (bf16) into the swizzled K-major operand: row r, 16-byte chunk c at
    // chunk c ^ (r % 8) of the row.
    {
      uint8_t* prow = p_smem + r * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 w;
        w.x = pack_bf16x2(x[8 * c + 0], x[8 * c + 1]);
        w.y = pack_bf16x2(x[8 * c + 2], x[8 * c + 3]);
        w.z = pack_bf16x2(x[8 * c + 4], x[8 * c + 5]);
        w.w = pack_bf16x2(x[8 * c + 6], x[8 * c + 7]);
        *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = w;
      }
    }
    // Tokens past the end of the last tile: their V rows may hold anything
    // (even NaN), and 0 * NaN must not reach O.
    if (j == n_kv - 1 && kv_end < (j + 1) * kPrefillKv) {
      const int first = kv_end - j * kPrefillKv;
      const int nvec = (kPrefillKv - first) * 8;
      for (int sb = 0; sb < S::SUB; ++sb)
        for (int v = threadIdx.x; v < nvec; v += blockDim.x)
          reinterpret_cast<uint4*>(v_smem + sb * (kPrefillKv * 128) + first * 128)[v] =
              make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
    tc_fence_before_sync();
    __syncthreads();

    // O += P V.
    if (threadIdx.x == 0) {
      tc_fence_after_sync();
      const uint32_t p_addr = smem_u32(p_smem), v_addr = smem_u32(v_smem);
#pragma unroll
      for (int kk = 0; kk < kPrefillKv / 16; ++kk) {
        const uint64_t ad = umma_desc_sw128(p_addr + kk * 32, 16, 1024);
        const uint64_t bd = umma_desc_sw128(v_addr + kk * 16 * 128, kPrefillKv * 128, 1024);
        umma_bf16(tmem_o, ad, bd, kIdescO, (j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(bar_o);
    }
  }

  if (ok) {
    ok = mbar_wait_bounded(bar_o, (uint32_t)((n_kv - 1) & 1));
    if (__syncthreads_or(!ok)) ok = false;
  }
  if (ok) {
    tc_fence_after_sync();
    __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                          ((size_t)(q0 + i) * p.Hq + (size_t)kvh * G + g) * D;
    const float inv = 1.f / l_run;
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t ov[32];
      tmem_ld32(tmem_o + lane_base + cc * 32, ov);
      tmem_wait_ld();
      if (row_valid) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(ov[e + 0]) * inv, __uint_as_float(ov[e + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(ov[e + 2]) * inv, __uint_as_float(ov[e + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(ov[e + 4]) * inv, __uint_as_float(ov[e + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(ov[e + 6]) * inv, __uint_as_float(ov[e + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + cc * 32 + e) = w;
        }
      }
    }
  } else if (threadIdx.x == 0) {
    flag_error(PKV_DEVERR_TIMEOUT);
    s_abort = 1;
  }
  // Free TMEM once every warp is done with it (and, after a timeout, once the
  // MMAs issued so far have had their bounded chance to finish).
  if (!ok && threadIdx.x == 0) {
    mbar_wait_bounded(bar_s, 0);
    mbar_wait_bounded(bar_o, 0);
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, S::kCols);
  }
}

}  // namespace pkv
