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
  // Two-tile kernel: work item = ((b * nqt + qt) * Hkv + kvh), one pair of
  // query tiles of one KV head.  sched (or NULL) = {next item, items with
  // work, order[...] longest first} for the persistent launch.
  int nqt;
  int n_items;
  int* sched;
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
  launch_overlap_entry();
  using S = PrefillSmem<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar_q = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  uint64_t* bar_kv = bar_q + 1;  // [2]
  uint64_t* bar_s = bar_q + 3;
  uint64_t* bar_o = bar_q + 4;
  uint64_t* bar_done = bar_q + 5;  // after a timeout: every MMA issued so far is complete
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  if (cta_timed_out()) return;
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
    mbar_init(bar_done, 1);
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
  int n_issued = 0;  // K/V tiles whose loads thread 0 has issued
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
    n_issued = min(n_kv, 2);
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
    if (__syncthreads_or(!ok)) { ok = false; break; }  // the CTA agrees
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
      if (__syncthreads_or(!ok)) { ok = false; break; }  // the CTA agrees
      tc_fence_after_sync();
      if (threadIdx.x == 0 && j + 1 < n_kv) {
        prefill_issue_kv<D>(p, stage_ptr(st ^ 1), &tmK, &tmV, &bar_kv[st ^ 1], bt_row, kvh, j + 1,
                            kv_end, pol);
        n_issued = j + 2;
      }
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
  // Free TMEM and shared memory once every warp is done with them; after a
  // timeout, once the MMAs and the loads issued so far have had their bounded
  // chance to finish.
  if (!ok && threadIdx.x == 0) {
    umma_commit(bar_done);
    mbar_wait_bounded(bar_done, 0);
    mbar_wait_bounded(bar_q, 0);
    for (int jj = max(0, n_issued - 2); jj < n_issued; ++jj)
      mbar_wait_bounded(&bar_kv[jj & 1], (uint32_t)((jj >> 1) & 1));
  }
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, S::kCols);
  }
}

// ---------------------------------------------------------------------------
// Warp-specialised two-tile kernel (D = 64 or 128).
//
// One CTA owns two query tiles of 128 rows (tile 0 = query tokens i0 ..
// i0 + TQ - 1, tile 1 = the next TQ) of one KV head, so every K/V tile brought
// into shared memory serves 256 rows.  Roles:
//  * warps 0-3 / 4-7: the softmax of tile 0 / tile 1 (thread = row);
//  * warp 8: the producer (TMA: both query tiles, then K_0, V_0, K_1, ... into
//    a ring of kRing slots, each one K or V tile);
//  * warp 9: the MMA issuer (one lane) and TMEM owner; warps 10-11 idle.
// The three warpgroups launch with 168 registers a thread; the third gives up
// all but kPpRegsIo and the two softmax warpgroups take kPpRegsSoftmax
// (2 x 128 x 200 + 128 x 96 <= 384 x 168).
//
// K/V tiles are 128 tokens.  TMEM (512 columns): S of tile t at 128 t, O of
// tile t at 256 + D t.  The softmax of tile t reads S (fp32), writes P as bf16
// pairs over the first 64 columns of the same S region, and the P V MMA takes
// P straight from TMEM.  MMA order per KV tile j:  P0 V_j, S0(j+1), P1 V_j,
// S1(j+1).  S_t(j+1) overwrites the columns P_t(j) V_j reads, so the issuer
// waits for that P V to complete first (while the other tile's MMA keeps the
// tensor pipe busy).  The softmax of tile 0 thus overlaps P1 V_{j-1} and
// S1(j), and tile 1 overlaps P0 V_j and S0(j+1).
// The running maximum only moves when a tile's maximum exceeds it by more than
// 2^8 (scores in log2 units), so O is rescaled rarely; P then stays below 256,
// and the final O / l is the same quotient.
// ---------------------------------------------------------------------------
constexpr int kPpKv = 128;          // tokens per K/V tile (MMA N of S, K of P V)
constexpr int kPpThreads = 384;     // 3 warpgroups
constexpr float kPpRescale = 8.0f;  // log2 growth of the row max that forces a rescale
constexpr uint32_t kPpRegsSoftmax = 200;
constexpr uint32_t kPpRegsIo = 96;
static_assert(2 * 128 * kPpRegsSoftmax + 128 * kPpRegsIo <= kPpThreads * 168,
              "register split exceeds the launch allocation");

template <int D>
struct PpSmem {
  static constexpr int SUB = D / 64;
  static constexpr int kRing = D == 64 ? 8 : 4;
  static constexpr int kQTile = SUB * kPrefillRows * 128;  // one query tile
  static constexpr int kKvTile = SUB * kPpKv * 128;        // one K or V tile
  static_assert(kKvTile % 1024 == 0, "ring slots keep the 1024-byte swizzle alignment");
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = 2 * kQTile;
  static constexpr int kOffBar = kOffRing + kRing * kKvTile;
  // q_full, q_empty, kv_full[kRing], kv_empty[kRing], s_full[2], p_full[2],
  // o_full[2], item_full[2], item_empty[2], done
  static constexpr int kNumBars = 2 + 2 * kRing + 11;
  static constexpr size_t kBytes = 1024 + (size_t)kOffBar + 8 * kNumBars;
  static_assert(kBytes <= 227 * 1024, "shared memory");
  static constexpr uint32_t kSCol = 0, kOCol = 256;  // + 128 t, + D t; P over S
  static constexpr uint32_t kCols = 512;
};

// Bounded wait that also gives up as soon as another role of the CTA has.
__device__ __forceinline__ bool pp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort = 1;
      flag_error(PKV_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// The same, agreed by the whole warp (so that warp-collective instructions
// after it are reached by all lanes or by none).
__device__ __forceinline__ bool pp_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return __all_sync(kFull, pp_wait(bar, parity, abort));
}

// Arrive once for the warp, after its tensor-memory accesses are complete.
__device__ __forceinline__ void pp_warp_arrive(uint64_t* bar) {
  tc_fence_before_sync();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}


// One K/V tile of the row softmax for the thread's row: read S_t(j), compute P
// and the running max / sum, rescale O if the max moved (the issuer computed
// S_t(j) only after P_t(j-1) V_{j-1} was done, so O is final), and write P
// over S.  After the first tile the exponentials are taken against the running
// maximum at once, and the tile's largest exponent is found in the same pass
// (it fills issue slots of a loop bound by the exponential unit); only a row
// whose maximum grew by more than kPpRescale takes the new one, and its warp
// reads S again.  Measured on B200 (chunked-append workload): 935-956 ->
// 966-968 TFLOP/s against a separate maximum pass.
template <int D>
__device__ __forceinline__ void pp_softmax_tile(uint32_t s_tm, uint32_t o_tm, int j, int visible,
                                                float cl2, bool pos, float& m_run, float& l_run) {
  const int tbase = j * kPpKv;
  // Reductions run over kAcc independent partial results (a tree, not a chain).
  constexpr int kAcc = 8;
  const bool masked = tbase + kPpKv > visible;
  const bool take_max = masked || pos;  // masked scores are already scaled
  const float k = masked ? 1.f : cl2;   // multiplier of x in the exponent
  float x[kPpKv];
  // S of this thread's row (warp-collective TMEM loads), scaled and masked on a
  // tile that crosses the row's causal limit.
  auto load_s = [&]() {
    uint32_t sv[4][32];
#pragma unroll
    for (int c = 0; c < 4; ++c) tmem_ld32(s_tm + c * 32, sv[c]);
    tmem_wait_ld();
#pragma unroll
    for (int c = 0; c < kPpKv; ++c) x[c] = __uint_as_float(sv[c / 32][c % 32]);
    if (masked) {
#pragma unroll
      for (int c = 0; c < kPpKv; ++c) x[c] = tbase + c < visible ? x[c] * cl2 : -INFINITY;
    }
  };
  load_s();
  uint32_t pk[2][32];
  float2 acc[kAcc / 2];
  float part[kAcc];
  // Exponentials of x * k - m, their sum and bf16 pairs; also the largest exponent.
  auto exps = [&](float m) {
    const float2 kk2 = make_float2(k, k), nm2 = make_float2(-m, -m);
#pragma unroll
    for (int a = 0; a < kAcc / 2; ++a) acc[a] = make_float2(0.f, 0.f);
#pragma unroll
    for (int a = 0; a < kAcc; ++a) part[a] = -INFINITY;
#pragma unroll
    for (int c = 0; c < kPpKv; c += 2) {
      const float2 e = ffma2(make_float2(x[c], x[c + 1]), kk2, nm2);
      part[(c / 2) % kAcc] = fmax3(part[(c / 2) % kAcc], e.x, e.y);
      float2 pr;
      pr.x = ex2_approx(e.x);
      pr.y = ex2_approx(e.y);
      acc[(c / 2) % (kAcc / 2)] = fadd2(acc[(c / 2) % (kAcc / 2)], pr);
      pk[c / 64][(c % 64) / 2] = pack_bf16x2(pr.x, pr.y);
    }
#pragma unroll
    for (int w = kAcc / 2; w > 0; w /= 2)
#pragma unroll
      for (int a = 0; a < w; ++a) part[a] = fmaxf(part[a], part[a + w]);
    return part[0];
  };
  float alpha = 1.f;
  if (j == 0) {
    // First tile: its maximum first (there is no running one yet), a tree of
    // 3-input max (or min, for a negative scale) over x.
#pragma unroll
    for (int a = 0; a < kAcc; ++a) part[a] = x[a];
    if (take_max) {
#pragma unroll
      for (int c = kAcc; c < kPpKv; c += 2 * kAcc)
#pragma unroll
        for (int a = 0; a < kAcc; ++a)
          part[a] = fmax3(part[a], x[c + a], x[c + kAcc + a < kPpKv ? c + kAcc + a : c + a]);
    } else {
#pragma unroll
      for (int c = kAcc; c < kPpKv; c += 2 * kAcc)
#pragma unroll
        for (int a = 0; a < kAcc; ++a)
          part[a] = fmin3(part[a], x[c + a], x[c + kAcc + a < kPpKv ? c + kAcc + a : c + a]);
    }
#pragma unroll
    for (int w = kAcc / 2; w > 0; w /= 2)
#pragma unroll
      for (int a = 0; a < w; ++a)
        part[a] = take_max ? fmaxf(part[a], part[a + w]) : fminf(part[a], part[a + w]);
    const float m_tile = masked ? part[0] : part[0] * k;
    alpha = ex2_approx(m_run - m_tile);
    m_run = m_tile;
    exps(m_run);
  } else {
    // Later tiles: the exponentials against the running maximum straight away,
    // the largest exponent beside them.  P stays below 2^kPpRescale unless a score
    // exceeds the running maximum by more; such a row takes the new maximum, and
    // the warp reads S again (it is still in TMEM) and exponentiates it again.
    const float e_max = exps(m_run);
    const bool grow = e_max > kPpRescale;
    if (__any_sync(kFull, grow)) {
      if (grow) {
        alpha = ex2_approx(-e_max);
        m_run += e_max;
      }
      load_s();
      exps(m_run);
    }
  }
#pragma unroll
  for (int w = kAcc / 4; w > 0; w /= 2)
#pragma unroll
    for (int a = 0; a < w; ++a) acc[a] = fadd2(acc[a], acc[a + w]);
  l_run = l_run * alpha + (acc[0].x + acc[0].y);
  if (j > 0 && __any_sync(kFull, alpha != 1.f)) {
#pragma unroll 1
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t ov[32];
      tmem_ld32(o_tm + cc * 32, ov);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
      tmem_st32(o_tm + cc * 32, ov);
    }
  }
  tmem_st32(s_tm + 0, pk[0]);
  tmem_st32(s_tm + 32, pk[1]);
  tmem_wait_st();
}

// One work item of the two-tile kernel: which rows, which tokens they see.
struct PpItem {
  int b, kvh, q0, Q, i0, ctx, kv_end, n_kv;  // n_kv = 0: nothing to do
  bool bad_len;                              // L > the table's capacity or Q > L
};

__device__ __forceinline__ PpItem pp_item(const PrefillParams& p, int item) {
  PpItem it{};
  it.kvh = item % p.Hkv;
  const int r = item / p.Hkv;
  const int qt = r % p.nqt;
  it.b = r / p.nqt;
  it.q0 = p.cu_q[it.b];
  it.Q = p.cu_q[it.b + 1] - it.q0;
  it.i0 = qt * 2 * p.TQ;
  it.n_kv = 0;
  int L = p.seq_lens[it.b];
  const int Lcap = min(p.max_blocks * p.bs, p.max_seq_len);
  it.bad_len = L > Lcap || it.Q > L;
  if (it.i0 >= it.Q || it.Q > min(L, Lcap)) return it;  // no rows, or no consistent reading
  L = min(L, Lcap);
  it.ctx = L - it.Q;
  it.kv_end = it.ctx + min(it.Q, it.i0 + 2 * p.TQ);  // tokens any row of the item sees
  it.n_kv = (it.kv_end + kPpKv - 1) / kPpKv;
  return it;
}

// Orders the work items for the persistent launch, which takes them in that order
// from an atomic counter.  The items of one (sequence, KV head) read the same K/V
// tiles, so they are kept together: the units are sorted longest first (a
// counting sort on the K/V tile count of a unit's longest item, ceil(L / 128),
// one block of kSchedThreads threads), and each unit's items follow one another,
// longest first.  Consecutive items start on different CTAs at about the same time
// and stream the same tiles together, so all but the first read of a tile are L2
// hits, while the longest units still start first and the short ones fill the
// tail.  Also flags bad lengths.
constexpr int kSchedThreads = 1024;  // = number of buckets

// A unit's items with work (qt < n, longest at qt = n - 1) and its bucket: thread
// order is descending cost.  n = 0 when no item of the unit has work.
__device__ __forceinline__ void prefill_unit(const PrefillParams& p, int b, int& n, int& bucket,
                                             bool& bad) {
  const int Q = p.cu_q[b + 1] - p.cu_q[b];
  const int L = p.seq_lens[b];
  const int Lcap = min(p.max_blocks * p.bs, p.max_seq_len);
  bad = L > Lcap || Q > L;
  n = 0;
  bucket = 0;
  if (Q <= 0 || Q > min(L, Lcap)) return;  // no rows, or no consistent reading
  n = min((Q + 2 * p.TQ - 1) / (2 * p.TQ), p.nqt);
  const int n_kv = (min(L, Lcap) + kPpKv - 1) / kPpKv;  // the last item sees every token
  bucket = kSchedThreads - 1 - min(n_kv, kSchedThreads - 1);
}

__global__ void __launch_bounds__(kSchedThreads)
    prefill_schedule_kernel(const PrefillParams p) {
  launch_overlap_entry();
  __shared__ int hist[kSchedThreads];
  __shared__ int warp_sum[kSchedThreads / 32];
  __shared__ int n_work;
  const int tid = threadIdx.x;
  const int n_units = p.n_items / p.nqt;  // (sequence, KV head) pairs
  hist[tid] = 0;
  if (tid == 0) n_work = 0;
  __syncthreads();
  for (int u = tid; u < n_units; u += kSchedThreads) {
    int n, bucket;
    bool bad;
    prefill_unit(p, u / p.Hkv, n, bucket, bad);
    if (bad && u % p.Hkv == 0) flag_error(PKV_DEVERR_SEQLEN);
    if (n > 0) {
      atomicAdd(&hist[bucket], n);
      atomicAdd(&n_work, n);
    }
  }
  __syncthreads();
  // Exclusive scan of hist in thread order.
  const int v = hist[tid];
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d *= 2) {
    const int y = __shfl_up_sync(kFull, incl, d);
    if ((tid & 31) >= d) incl += y;
  }
  if ((tid & 31) == 31) warp_sum[tid / 32] = incl;
  __syncthreads();
  if (tid < 32) {
    int w = warp_sum[tid];
#pragma unroll
    for (int d = 1; d < 32; d *= 2) {
      const int y = __shfl_up_sync(kFull, w, d);
      if (tid >= d) w += y;
    }
    warp_sum[tid] = w;  // inclusive over warps
  }
  __syncthreads();
  hist[tid] = incl - v + (tid >= 32 ? warp_sum[tid / 32 - 1] : 0);
  __syncthreads();
  int* order = p.sched + 2;
  for (int u = tid; u < n_units; u += kSchedThreads) {
    int n, bucket;
    bool bad;
    const int b = u / p.Hkv, kvh = u % p.Hkv;
    prefill_unit(p, b, n, bucket, bad);
    if (n > 0) {
      int at = atomicAdd(&hist[bucket], n);
      for (int qt = n - 1; qt >= 0; --qt) order[at++] = (b * p.nqt + qt) * p.Hkv + kvh;
    }
  }
  if (tid == 0) {
    p.sched[0] = 0;
    p.sched[1] = n_work;
  }
}

// Persistent (or one item per CTA) two-tile kernel.  The producer takes work
// items (from the ordered list when p.sched is set, else the CTA's own item)
// and passes them to the other roles through a two-deep queue in shared
// memory; it runs ahead into the next item's query and K/V tiles while the
// current one finishes.  Barrier phases follow per-CTA counters of items (k)
// and of K/V tiles (g), so they carry over from one item to the next.
template <int D>
__global__ void __launch_bounds__(kPpThreads, 1)
    paged_prefill_pp_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmK,
                            const __grid_constant__ CUtensorMap tmV) {
  launch_overlap_entry();
  using S = PpSmem<D>;
  constexpr int R = S::kRing;
  constexpr int kBoxes = kPpKv / kStageTokens;  // 16-token boxes per K/V tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;
  uint64_t* kv_empty = bars + 2 + R;
  uint64_t* s_full = bars + 2 + 2 * R;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = s_full + 4;
  uint64_t* item_full = s_full + 6;
  uint64_t* item_empty = s_full + 8;
  uint64_t* done = s_full + 10;
  __shared__ uint32_t s_tmem;
  __shared__ volatile int s_abort;
  __shared__ int s_item[2];

  if (cta_timed_out()) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G, TQ = p.TQ;
  const bool persistent = p.sched != nullptr;
  int own_item = -1;
  if (!persistent) {
    // One item per CTA: the longest query tiles of a sequence first.
    own_item = ((int)blockIdx.z * p.nqt + (p.nqt - 1 - (int)blockIdx.y)) * p.Hkv + (int)blockIdx.x;
    const PpItem it = pp_item(p, own_item);
    if (threadIdx.x == 0 && it.bad_len && it.i0 == 0 && it.kvh == 0) flag_error(PKV_DEVERR_SEQLEN);
    if (it.n_kv == 0) return;
  }

  if (warp == 9) {
    tmem_alloc(&s_tmem, S::kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < R; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 4);  // one arrival per softmax warp
      mbar_init(&o_full[t], 1);
      mbar_init(&item_full[t], 1);
      mbar_init(&item_empty[t], 9);  // 8 softmax warps + the MMA warp
    }
    mbar_init(done, 1);
    fence_mbar_init();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = s_tmem;
  uint8_t* q_smem = smem + S::kOffQ;
  uint8_t* ring = smem + S::kOffRing;
  if (warp < 8) regs_inc<kPpRegsSoftmax>();
  else regs_dec<kPpRegsIo>();

  // Consumers: the next item from the queue (-1: no more), released at once.
  auto pop_item = [&](int k, int& item) -> bool {
    if (!pp_wait_warp(&item_full[k & 1], (uint32_t)((k >> 1) & 1), &s_abort)) return false;
    item = *reinterpret_cast<volatile int*>(&s_item[k & 1]);
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[k & 1]);
    return true;
  };

  if (warp < 8) {
    // ---- softmax of tile t = warp / 4; thread = row r ----
    const int t = warp / 4;
    const int r = threadIdx.x % 128;
    const uint32_t lane_base = (uint32_t)((warp % 4) * 32) << 16;
    const uint32_t s_tm = tmem + S::kSCol + 128u * t + lane_base;
    const uint32_t o_tm = tmem + S::kOCol + (uint32_t)D * t + lane_base;
    const float cl2 = p.scale_log2;
    const bool pos = cl2 >= 0.f;
    int g = 0;  // K/V tiles before this item
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item;
      if (!(ok = pop_item(k, item)) || item < 0) break;
      const PpItem it = pp_item(p, item);
      const int i = it.i0 + t * TQ + r / G, gh = r % G;
      const bool row_valid = i < it.Q;
      const int visible = min(it.ctx + i + 1, it.kv_end);
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < it.n_kv; ++j) {
        if (!(ok = pp_wait_warp(&s_full[t], (uint32_t)((g + j) & 1), &s_abort))) break;
        tc_fence_after_sync();
        pp_softmax_tile<D>(s_tm, o_tm, j, visible, cl2, pos, m_run, l_run);
        pp_warp_arrive(&p_full[t]);
      }
      if (ok) ok = pp_wait_warp(&o_full[t], (uint32_t)((g + it.n_kv - 1) & 1), &s_abort);
      if (!ok) break;
      tc_fence_after_sync();
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) +
                            ((size_t)(it.q0 + i) * p.Hq + (size_t)it.kvh * G + gh) * D;
      const float inv = 1.f / l_run;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t ov[32];
        tmem_ld32(o_tm + cc * 32, ov);
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
      g += it.n_kv;
    }
  } else if (warp == 8) {
    // ---- producer ----
    const uint64_t pol = l2_policy_evict_first();
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
    }
    int kv_idx = 0;   // K/V ring loads issued so far (K and V of each tile)
    int q_loads = 0;  // query tile pairs issued so far
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item = -1;
      if (persistent) {
        if (lane == 0) {
          const int n = atomicAdd(p.sched, 1);
          item = n < p.sched[1] ? p.sched[2 + n] : -1;
        }
        item = __shfl_sync(kFull, item, 0);
      } else {
        item = k == 0 ? own_item : -1;
      }
      if (!(ok = pp_wait_warp(&item_empty[k & 1], (uint32_t)(((k >> 1) & 1) ^ 1), &s_abort))) break;
      if (lane == 0) {
        s_item[k & 1] = item;
        mbar_arrive(&item_full[k & 1]);  // release: the store above is seen with the phase
      }
      if (item < 0) break;
      const PpItem it = pp_item(p, item);
      // The query tiles, once the previous item's last S MMA has read the old ones.
      if (k > 0 && !(ok = pp_wait_warp(q_empty, (uint32_t)((k - 1) & 1), &s_abort))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, 2 * S::kQTile);
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
          for (int sb = 0; sb < S::SUB; ++sb)
            tma_load_3d(q_smem + t * S::kQTile + sb * (kPrefillRows * 128), &tmQ, q_full,
                        sb * 64, it.kvh * G, it.q0 + it.i0 + t * TQ, pol);
      }
      ++q_loads;
      const int32_t* bt_row = p.block_tables + (size_t)it.b * p.max_blocks;
      int row = p.num_blocks * p.bs;  // box row of this lane's 16 tokens (past the end: zeros)
      for (int e = 0; e < 2 * it.n_kv; ++e, ++kv_idx) {
        const int j = e >> 1, slot = kv_idx % R;
        if ((e & 1) == 0 && lane < kBoxes) {
          const int t0 = j * kPpKv + lane * kStageTokens;
          row = p.num_blocks * p.bs;
          if (t0 < it.kv_end) {
            const int id = bt_row[t0 / p.bs];
            if (id >= 0 && id < p.num_blocks) row = id * p.bs + t0 % p.bs;
            else flag_error(PKV_DEVERR_BLOCK_ID);
          }
        }
        if (!(ok = pp_wait_warp(&kv_empty[slot], (uint32_t)(((kv_idx / R) & 1) ^ 1), &s_abort))) break;
        if (lane == 0) mbar_arrive_expect_tx(&kv_full[slot], S::kKvTile);
        __syncwarp();
        if (lane < kBoxes) {
          const CUtensorMap* map = (e & 1) ? &tmV : &tmK;
#pragma unroll
          for (int sb = 0; sb < S::SUB; ++sb)
            tma_load_3d(ring + slot * S::kKvTile + sb * (kPpKv * 128) + lane * (kStageTokens * 128),
                        map, &kv_full[slot], sb * 64, it.kvh, row, pol);
        }
      }
    }
    // Loads still in flight after an abort land before the CTA lets go of its
    // shared memory (bounded).
    if (s_abort && lane == 0) {
      for (int idx = max(0, kv_idx - R); idx < kv_idx; ++idx)
        mbar_wait_bounded(&kv_full[idx % R], (uint32_t)((idx / R) & 1));
      if (q_loads > 0) mbar_wait_bounded(q_full, (uint32_t)((q_loads - 1) & 1));
    }
  } else if (warp == 9) {
    // ---- MMA issuer ----
    constexpr uint32_t kIdescS = umma_idesc_bf16(kPrefillRows, kPpKv, false);
    constexpr uint32_t kIdescO = umma_idesc_bf16(kPrefillRows, D, true);
    const bool leader = lane == 0;
    // Descriptors of the smem bases; an operand at byte offset o is base + o / 16
    // (all of shared memory is below 2^18 bytes, so the 14-bit address field
    // never carries).
    const uint64_t q_desc = umma_desc_sw128(smem_u32(q_smem), 16, 1024);
    const uint64_t k_desc = umma_desc_sw128(smem_u32(ring), 16, 1024);
    const uint64_t v_desc = umma_desc_sw128(smem_u32(ring), kPpKv * 128, 1024);
    auto issue_s = [&](int t, int kslot) {
      const uint64_t qd = q_desc + (uint64_t)((t * S::kQTile) >> 4);
      const uint64_t kd = k_desc + (uint64_t)((kslot * S::kKvTile) >> 4);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t ad = qd + (uint64_t)(((kk / 4) * (kPrefillRows * 128) + (kk % 4) * 32) >> 4);
        const uint64_t bd = kd + (uint64_t)(((kk / 4) * (kPpKv * 128) + (kk % 4) * 32) >> 4);
        umma_bf16(tmem + S::kSCol + 128u * t, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
      }
      umma_commit(&s_full[t]);
    };
    auto issue_pv = [&](int t, int vslot, bool first) {
      const uint64_t vd = v_desc + (uint64_t)((vslot * S::kKvTile) >> 4);
#pragma unroll
      for (int kk = 0; kk < kPpKv / 16; ++kk) {
        umma_bf16_tmem_a(tmem + S::kOCol + (uint32_t)D * t, tmem + S::kSCol + 128u * t + 8u * kk,
                         vd + (uint64_t)((kk * 16 * 128) >> 4), kIdescO, (!first || kk > 0) ? 1u : 0u);
      }
      umma_commit(&o_full[t]);
    };
    int g = 0, kv_idx = 0;
    bool ok = true;
    for (int k = 0; ok; ++k) {
      int item;
      if (!(ok = pop_item(k, item)) || item < 0) break;
      const PpItem it = pp_item(p, item);
      const int n = it.n_kv;
      // S(0) of both tiles, once the query tiles and K_0 are in and (from the
      // second item on) the previous P V has read the S / P columns.
      if (!(ok = pp_wait_warp(q_full, (uint32_t)(k & 1), &s_abort))) break;
      if (!(ok = pp_wait_warp(&kv_full[kv_idx % R], (uint32_t)((kv_idx / R) & 1), &s_abort))) break;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if (g > 0 && !(ok = pp_wait_warp(&o_full[t], (uint32_t)((g - 1) & 1), &s_abort))) break;
        tc_fence_after_sync();
        if (leader) {
          issue_s(t, kv_idx % R);
          if (t == 1) {
            umma_commit(&kv_empty[kv_idx % R]);
            if (n == 1) umma_commit(q_empty);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      for (int j = 0; ok && j < n; ++j) {
        const int iv = kv_idx + 2 * j + 1, ik = kv_idx + 2 * j + 2;
        if (!(ok = pp_wait_warp(&kv_full[iv % R], (uint32_t)((iv / R) & 1), &s_abort))) break;
        if (j == n - 1 && it.kv_end < n * kPpKv) {
          // Tokens past the end: their V rows may hold anything (even NaN), and
          // 0 * NaN must not reach O.
          uint8_t* v_smem = ring + (iv % R) * S::kKvTile;
          const int first = it.kv_end - j * kPpKv;
          const int nvec = (kPpKv - first) * 8;
          for (int sb = 0; sb < S::SUB; ++sb)
            for (int v = lane; v < nvec; v += 32)
              reinterpret_cast<uint4*>(v_smem + sb * (kPpKv * 128) + first * 128)[v] =
                  make_uint4(0u, 0u, 0u, 0u);
          fence_proxy_async_smem();
          __syncwarp();
        }
        if (j + 1 < n && !(ok = pp_wait_warp(&kv_full[ik % R], (uint32_t)((ik / R) & 1), &s_abort)))
          break;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          // P_t V_j, then S_t(j+1) over the columns it read once it is done.
          if (!(ok = pp_wait_warp(&p_full[t], (uint32_t)((g + j) & 1), &s_abort))) break;
          tc_fence_after_sync();
          if (leader) {
            issue_pv(t, iv % R, j == 0);
            if (t == 1) umma_commit(&kv_empty[iv % R]);
          }
          __syncwarp();
          if (j + 1 < n) {
            if (!(ok = pp_wait_warp(&o_full[t], (uint32_t)((g + j) & 1), &s_abort))) break;
            tc_fence_after_sync();
            if (leader) {
              issue_s(t, ik % R);
              if (t == 1) {
                umma_commit(&kv_empty[ik % R]);
                if (j + 2 == n) umma_commit(q_empty);  // the item's last S
              }
            }
            __syncwarp();
          }
        }
      }
      g += n;
      kv_idx += 2 * n;
    }
    // Every MMA issued has finished before TMEM is released (bounded).
    if (leader) {
      umma_commit(done);
      mbar_wait_bounded(done, 0);
    }
    __syncwarp();
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after_sync();
    tmem_dealloc(tmem, S::kCols);
  }
}

}  // namespace pkv
