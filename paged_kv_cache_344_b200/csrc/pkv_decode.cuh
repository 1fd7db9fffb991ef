// Decode-step attention over a block-paged KV cache (sm_100a).
//
// What is computed: for sequence b and query head h (KV head kvh = h / G),
//   out[b][h] = sum_t softmax_t(scale * q[b][h] . K_t) V_t,  t < seq_lens[b],
// with K_t, V_t found through the block table: logical block t / block_size,
// offset t % block_size ("Paged Attention Explained", Step 3 and Step 4;
// "PagedAttention: paging the KV cache like an OS pages memory", How it works:
// the attention is ordinary softmax attention, only the layout changes).
//
// How (B200 design):
//  * one CTA per (kvh, partition, b); the G query heads of a KV head share
//    every K/V byte read, so the cache is read once per (b, kvh);
//  * K/V arrive by TMA, one 16-token slab of one KV head per box (a 4-D map
//    with the 128-byte swizzle for the tensor-core consumer, a 3-D map for the
//    CUDA-core one; with 8-token blocks a stage is two 8-token boxes from two
//    blocks); each consumer warp owns a ring of stages and refills it itself,
//    so no CTA-wide barrier sits in the loop;
//  * the block-table walk (the "pointer chase") is taken off the critical path:
//    each warp keeps the physical ids of its next 32..64 stages in registers.
//    The unpaged control (kLayoutContig) reads [B][stride][Hkv][D] with no
//    table at all, to measure what the walk costs;
//  * online softmax in fp32 (running max and sum, exp2 with the scale folded
//    into log2 units), per warp; warps and then partitions are merged with a
//    log-sum-exp rescale;
//  * bf16 runs the score and PV products on the tensor cores with a
//    warp-level m16n8k16 MMA: tokens are M, the G heads of a KV head are N
//    (padded to 8), D is K; PV computes O^T = V^T P^T with P transposed in
//    registers by movmatrix.  fp32 (and, on request, bf16) uses CUDA-core FMAs;
//  * a sequence split into several partitions writes partial (max, sum,
//    weighted V) to the workspace; the CTA that finishes last for a
//    (b, kvh) -- found with an atomic ticket, no spinning -- merges them.
#pragma once

#include "pkv_ptx.cuh"

namespace pkv {

constexpr int kStageTokens = 16;  // tokens per TMA box / pipeline stage
constexpr int kWarps = 4;         // consumer warps per CTA
constexpr uint32_t kFull = 0xffffffffu;

__device__ uint32_t g_device_errors;  // OR of PKV_DEVERR_* bits

__device__ __forceinline__ void flag_error(uint32_t bits) { atomicOr(&g_device_errors, bits); }

// True once a pipeline wait has timed out anywhere on the device.  Thread 0 reads
// the flag and one barrier hands its answer to the whole CTA, so a CTA stops whole
// or runs whole: no barrier further on can miss a warp that returned early.
__device__ __forceinline__ bool cta_timed_out() {
  const bool t = threadIdx.x == 0 &&
                 (*reinterpret_cast<volatile uint32_t*>(&g_device_errors) & PKV_DEVERR_TIMEOUT);
  return __syncthreads_or(t) != 0;
}

struct DecodeParams {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float* ws_acc;       // [B*Hkv*max_parts*G][D]
  float2* ws_ml;       // [B*Hkv*max_parts*G] (max in log2 units, sum)
  uint32_t* ws_count;  // [B*Hkv] finished-partition tickets
  int B;
  int max_blocks;
  int max_seq_len;
  int Hq;
  int Hkv;
  int G;
  int bs;
  int part_tokens;
  int max_parts;
  int num_blocks;
  float scale_log2;  // scale * log2(e)
  // Fused step (paged_decode_step): the CTA of a sequence's last partition first
  // copies the copy-on-write source block and writes the new token (position
  // L - 1), both for its own KV head.  Null k_new: plain decode.
  const void* k_new;     // [B][Hkv][D]
  const void* v_new;
  void* k_cache_w;       // the caches, written by the fused step
  void* v_cache_w;
  const int32_t* cow_src;  // [B] or null: block copied into the new token's block first
  // Nonzero: CTAs take their (sequence, partition, KV head) in length order
  // (sorted_item) instead of from their grid coordinates.
  int sorted;
};

template <typename T>
__device__ __forceinline__ T to_out(float x);
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <>
__device__ __forceinline__ float to_out<float>(float x) {
  return x;
}

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& w, float* f);
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& w, float* f) {
  f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x); f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
  f[4] = bf16_lo(w.z); f[5] = bf16_hi(w.z); f[6] = bf16_lo(w.w); f[7] = bf16_hi(w.w);
}
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& w, float* f) {
  f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
  f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
}

// Loads N consecutive elements of type T from shared memory as floats.
template <typename T, int N>
__device__ __forceinline__ void load_row_slice(const uint8_t* src, float* f) {
  constexpr int BYTES = N * (int)sizeof(T);
  if constexpr (BYTES == 16) {
    unpack16<T>(*reinterpret_cast<const uint4*>(src), f);
  } else if constexpr (BYTES == 8) {
    const uint2 w = *reinterpret_cast<const uint2*>(src);
    if constexpr (sizeof(T) == 2) {
      f[0] = bf16_lo(w.x); f[1] = bf16_hi(w.x); f[2] = bf16_lo(w.y); f[3] = bf16_hi(w.y);
    } else {
      f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
    }
  } else if constexpr (BYTES == 4) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(src);
    if constexpr (sizeof(T) == 2) {
      f[0] = bf16_lo(w); f[1] = bf16_hi(w);
    } else {
      f[0] = __uint_as_float(w);
    }
  } else {
    static_assert(BYTES == 32, "unsupported slice");
    unpack16<T>(*reinterpret_cast<const uint4*>(src), f);
    unpack16<T>(*reinterpret_cast<const uint4*>(src + 16), f + 16 / sizeof(T));
  }
}

// ---------------------------------------------------------------------------
// CUDA-core consumer: one warp processes a 16-token stage.  QK: LPT lanes per
// token, each lane two 16-byte chunks of the K row; PV: each lane D/32
// consecutive dims of every V row.
// ---------------------------------------------------------------------------
template <typename T, int D, int GMAX>
struct SimtConsumer {
  static constexpr int ES = sizeof(T);
  static constexpr int ROWB = D * ES;
  static constexpr int CH = ROWB / 16;
  static constexpr int LPT = CH / 2;
  static constexpr int TPI = 32 / LPT;
  static constexpr int ITERS = kStageTokens / TPI;
  static constexpr int EPC = 16 / ES;
  static constexpr int DPL = D / 32;
  static constexpr int kTileBytes = kStageTokens * ROWB;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = ROWB <= 128 ? 6 : (ROWB <= 256 ? 3 : 2);
  static constexpr int GP = GMAX;
  static constexpr bool kSwizzle = false;
  static_assert(LPT >= 1 && LPT <= 32 && TPI * LPT == 32, "bad lane split");

  float qv[GMAX][2][EPC];
  float m[GMAX], l[GMAX], acc[GMAX][DPL];

  __device__ __forceinline__ void init(const DecodeParams& p, int b, int kvh, int lane) {
    const int sub = lane % LPT;
    const T* q = reinterpret_cast<const T*>(p.q);
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < p.G) {
        const T* row = q + ((size_t)b * p.Hq + (size_t)kvh * p.G + g) * D;
        unpack16<T>(*reinterpret_cast<const uint4*>(row + sub * EPC), qv[g][0]);
        unpack16<T>(*reinterpret_cast<const uint4*>(row + (sub + LPT) * EPC), qv[g][1]);
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
          qv[g][0][e] *= p.scale_log2;
          qv[g][1][e] *= p.scale_log2;
        }
      } else {
#pragma unroll
        for (int e = 0; e < EPC; ++e) qv[g][0][e] = qv[g][1][e] = 0.f;
      }
      m[g] = -INFINITY;
      l[g] = 0.f;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[g][e] = 0.f;
    }
  }

  static __device__ __forceinline__ void load_stage(uint8_t* st, const CUtensorMap* tk,
                                                    const CUtensorMap* tv, uint64_t* bar,
                                                    int kvh, int row, uint64_t pol) {
    tma_load_3d(st, tk, bar, 0, kvh, row, pol);
    tma_load_3d(st + kTileBytes, tv, bar, 0, kvh, row, pol);
  }

  // Blocks of 8 tokens: the stage's two halves come from two blocks (8-row boxes).
  static __device__ __forceinline__ void load_stage_halves(uint8_t* st, const CUtensorMap* tk,
                                                           const CUtensorMap* tv, uint64_t* bar,
                                                           int kvh, int row0, int row1,
                                                           uint64_t pol) {
    constexpr int kHalf = kStageTokens / 2 * ROWB;
    tma_load_3d(st, tk, bar, 0, kvh, row0, pol);
    tma_load_3d(st + kHalf, tk, bar, 0, kvh, row1, pol);
    tma_load_3d(st + kTileBytes, tv, bar, 0, kvh, row0, pol);
    tma_load_3d(st + kTileBytes + kHalf, tv, bar, 0, kvh, row1, pol);
  }

  // `release()` (warp-collective) is called once the stage's shared memory is no
  // longer needed; here that is after the whole stage.
  template <class Release>
  __device__ __forceinline__ void consume(uint8_t* st, int n_valid, int lane, Release&& release) {
    consume_body(st, n_valid, lane);
    __syncwarp();
    release();
  }

  __device__ __forceinline__ void consume_body(uint8_t* st, int n_valid, int lane) {
    const uint8_t* sk = st;
    const uint8_t* sv = st + kTileBytes;
    const int sub = lane % LPT;
    const int tg = lane / LPT;
    float s[ITERS][GMAX];
#pragma unroll
    for (int it = 0; it < ITERS; ++it) {
      const int tok = it * TPI + tg;
      float k0[EPC], k1[EPC];
      unpack16<T>(*reinterpret_cast<const uint4*>(sk + tok * ROWB + sub * 16), k0);
      unpack16<T>(*reinterpret_cast<const uint4*>(sk + tok * ROWB + (sub + LPT) * 16), k1);
#pragma unroll
      for (int g = 0; g < GMAX; ++g) {
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < EPC; ++e) part = fmaf(qv[g][0][e], k0[e], part);
#pragma unroll
        for (int e = 0; e < EPC; ++e) part = fmaf(qv[g][1][e], k1[e], part);
#pragma unroll
        for (int off = LPT / 2; off >= 1; off /= 2) part += __shfl_xor_sync(kFull, part, off);
        s[it][g] = (tok < n_valid) ? part : -INFINITY;
      }
    }
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      float mx = s[0][g];
#pragma unroll
      for (int it = 1; it < ITERS; ++it) mx = fmaxf(mx, s[it][g]);
#pragma unroll
      for (int off = LPT; off < 32; off *= 2) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, off));
      const float m_new = fmaxf(m[g], mx);
      const float alpha = exp2f(m[g] - m_new);
      m[g] = m_new;
      float sum = 0.f;
#pragma unroll
      for (int it = 0; it < ITERS; ++it) {
        s[it][g] = exp2f(s[it][g] - m_new);
        sum += s[it][g];
      }
#pragma unroll
      for (int off = LPT; off < 32; off *= 2) sum += __shfl_xor_sync(kFull, sum, off);
      l[g] = l[g] * alpha + sum;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[g][e] *= alpha;
    }
#pragma unroll
    for (int t = 0; t < kStageTokens; ++t) {
      if (t < n_valid) {
        float v[DPL];
        load_row_slice<T, DPL>(sv + t * ROWB + lane * DPL * ES, v);
#pragma unroll
        for (int g = 0; g < GMAX; ++g) {
          const float pt = __shfl_sync(kFull, s[t / TPI][g], (t % TPI) * LPT);
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[g][e] = fmaf(pt, v[e], acc[g][e]);
        }
      }
    }
  }

  // Per-warp state -> shared memory: m[GP], l[GP], acc[GP][D].
  __device__ __forceinline__ void store_state(float* dst, int lane) const {
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (lane == 0) {
        dst[g] = m[g];
        dst[GP + g] = l[g];
      }
#pragma unroll
      for (int e = 0; e < DPL; ++e) dst[2 * GP + g * D + lane * DPL + e] = acc[g][e];
    }
  }

  // Final rows out[g][d] = acc / l for g < G (rows of one KV head, contiguous).
  __device__ __forceinline__ void write_out(T* out, int G, int lane) const {
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < G) {
        const float inv = 1.f / l[g];
#pragma unroll
        for (int e = 0; e < DPL; ++e) out[g * D + lane * DPL + e] = to_out<T>(acc[g][e] * inv);
      }
    }
  }

  // Unnormalised partial: acc[g][d], and (max in log2 units, sum) per head.
  __device__ __forceinline__ void write_partial(float* acc_dst, float2* ml_dst, int G,
                                                int lane) const {
#pragma unroll
    for (int g = 0; g < GMAX; ++g) {
      if (g < G) {
        if (lane == 0) ml_dst[g] = make_float2(m[g], l[g]);
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc_dst[g * D + lane * DPL + e] = acc[g][e];
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Tensor-core consumer (bf16): S[t][g] = K[t][:] . Q[g][:] with tokens as M,
// heads as N; O^T[d][g] += V^T[d][t] P[t][g].  K/V tiles arrive with the TMA
// 128-byte swizzle (D/64 sub-tiles of 16 rows x 128 B), which keeps the
// ldmatrix row reads free of bank conflicts.
// ---------------------------------------------------------------------------
// Pipeline stages per warp of the tensor-core consumer at D = 128 (8 KB each).
// 2 stages give 66.6 KB of shared memory per CTA and 3 resident CTAs per SM
// (12 warps, 192 KB of loads in flight), which hides each CTA's start-up
// behind its neighbours.  Measured on B200 against 3 stages (2 CTAs per SM):
// equal on MHA and GQA, +3.6% on the long-context workload.
#ifndef PKV_MMA_STAGES_D128
#define PKV_MMA_STAGES_D128 2
#endif

template <int D, int NT, int STAGES = (D <= 64 ? 6 : (D <= 128 ? PKV_MMA_STAGES_D128 : 2)),
          bool EARLY = (D <= 128 && NT == 1)>
struct MmaConsumer {
  static constexpr int SUB = D / 64;
  static constexpr int kSubBytes = kStageTokens * 128;
  static constexpr int kTileBytes = SUB * kSubBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;
  static constexpr int kStages = STAGES;
  static constexpr int KS = D / 16;
  static constexpr int MT = D / 16;
  static constexpr int GP = 8 * NT;
  static constexpr bool kSwizzle = true;
  // V fragments held in registers so that the stage is released before the
  // softmax.  By default for one 8-row head tile up to D = 128: with two tiles (16
  // query rows) or D = 256 the extra registers cost a resident CTA per SM (or
  // spill), and measured on B200 the early release gains nothing there.
  static constexpr bool kEarly = EARLY;

  uint32_t qf[NT][KS][2];
  float m[NT][2], l[NT][2];
  float o[NT][MT][4];
  float scale_log2;

  __device__ __forceinline__ void init(const DecodeParams& p, int b, int kvh, int lane) {
    const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q);
    scale_log2 = p.scale_log2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + lane / 4;
      const uint32_t* row = reinterpret_cast<const uint32_t*>(
          q + ((size_t)b * p.Hq + (size_t)kvh * p.G + (g < p.G ? g : 0)) * D);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int d0 = ks * 16 + 2 * (lane % 4);
        qf[nt][ks][0] = g < p.G ? row[d0 / 2] : 0u;
        qf[nt][ks][1] = g < p.G ? row[(d0 + 8) / 2] : 0u;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m[nt][j] = -INFINITY;
        l[nt][j] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[nt][mt][j] = 0.f;
    }
  }

  // Rows n = i * G + g of the N dimension gather query head kvh * G + g of
  // sequence b0 + i, for i < members (the members of a shared-prefix group).
  __device__ __forceinline__ void init_gather(const DecodeParams& p, int b0, int members,
                                              int kvh, int lane) {
    const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p.q);
    scale_log2 = p.scale_log2;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int n = nt * 8 + lane / 4;
      const int i = n / p.G, g = n % p.G;
      const bool valid = i < members;
      const uint32_t* row = reinterpret_cast<const uint32_t*>(
          q + ((size_t)(b0 + (valid ? i : 0)) * p.Hq + (size_t)kvh * p.G + g) * D);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int d0 = ks * 16 + 2 * (lane % 4);
        qf[nt][ks][0] = valid ? row[d0 / 2] : 0u;
        qf[nt][ks][1] = valid ? row[(d0 + 8) / 2] : 0u;
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        m[nt][j] = -INFINITY;
        l[nt][j] = 0.f;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int j = 0; j < 4; ++j) o[nt][mt][j] = 0.f;
    }
  }

  // One box per tile: the stage maps are 4-D (64 dims, tokens, 64-dim halves,
  // KV heads), so a box of 16 tokens lands as SUB swizzled 16 x 128 B sub-tiles.
  static __device__ __forceinline__ void load_stage(uint8_t* st, const CUtensorMap* tk,
                                                    const CUtensorMap* tv, uint64_t* bar,
                                                    int kvh, int row, uint64_t pol) {
    tma_load_4d(st, tk, bar, 0, row, 0, kvh, pol);
    tma_load_4d(st + kTileBytes, tv, bar, 0, row, 0, kvh, pol);
  }

  // Blocks of 8 tokens: the maps' box is {64, 8, 1, 1}, and each 64-dim sub-tile is
  // filled by two boxes, rows 0..7 from the first block and 8..15 from the second.
  // The second box lands 1024 bytes in, where the 128-byte swizzle pattern repeats,
  // so the sub-tile reads exactly like one 16-row box.
  static __device__ __forceinline__ void load_stage_halves(uint8_t* st, const CUtensorMap* tk,
                                                           const CUtensorMap* tv, uint64_t* bar,
                                                           int kvh, int row0, int row1,
                                                           uint64_t pol) {
#pragma unroll
    for (int sb = 0; sb < SUB; ++sb) {
      uint8_t* k = st + sb * kSubBytes;
      uint8_t* v = k + kTileBytes;
      tma_load_4d(k, tk, bar, 0, row0, sb, kvh, pol);
      tma_load_4d(k + kSubBytes / 2, tk, bar, 0, row1, sb, kvh, pol);
      tma_load_4d(v, tv, bar, 0, row0, sb, kvh, pol);
      tma_load_4d(v + kSubBytes / 2, tv, bar, 0, row1, sb, kvh, pol);
    }
  }

  // Byte offset of (row, 16-byte chunk) inside a swizzled 16x128 B sub-tile.
  static __device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
  }

  // Consumes one stage; `release()` (warp-collective) is called as soon as the
  // stage's shared memory has been read: with kEarly after the score MMAs and the
  // V fragments' loads into registers, so that the warp refills the slot while it
  // still computes the softmax and the P V product; otherwise after the P V product.
  template <class Release>
  __device__ __forceinline__ void consume(uint8_t* st, int n_valid, int lane, Release&& release) {
    consume_impl<false>(st, n_valid, lane, 0, GP, release);
  }

  // The same, with only query rows [r0, r1) of the N dimension scoring this
  // stage (the others see it as masked): a stage of one member's own tokens in a
  // shared-prefix group.  A row may then have seen no token yet, so the
  // rescale factors are guarded against -inf - -inf.
  template <class Release>
  __device__ __forceinline__ void consume_rows(uint8_t* st, int n_valid, int lane, int r0, int r1,
                                               Release&& release) {
    consume_impl<true>(st, n_valid, lane, r0, r1, release);
  }

  template <bool kRows, class Release>
  __device__ __forceinline__ void consume_impl(uint8_t* st, int n_valid, int lane, int r0, int r1,
                                               Release& release) {
    const uint32_t sk = smem_u32(st);
    const uint32_t sv = sk + kTileBytes;
    const int mi = lane / 8, rr = lane % 8;
    // With a row range, 8-row tiles outside it are skipped altogether: their
    // state is what a fully masked stage would leave.
    auto live = [&](int nt) { return !kRows || (nt * 8 < r1 && nt * 8 + 8 > r0); };

    // Scores: S = K Q^T, one m16n8k16 per (k-step, head tile), the even and
    // the odd k-steps in two accumulators so that the MMA chain is half as long.
    float s[NT][4], s2[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[nt][j] = s2[nt][j] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const int row = rr + (mi & 1) * 8;
      const int chunk = (ks % 4) * 2 + (mi >> 1);
      uint32_t a[4];
      ldmatrix_x4(sk + (ks / 4) * kSubBytes + swz(row, chunk), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        if (live(nt)) mma_bf16_16816(ks % 2 ? s2[nt] : s[nt], a, qf[nt][ks][0], qf[nt][ks][1]);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[nt][j] += s2[nt][j];

    // V^T fragments (A operand of O^T += V^T P): lane (g, t) = (lane / 4, lane % 4)
    // holds dims (g, g + 8) of each 16-dim tile for tokens (2t, 2t + 1) in
    // va[mt][0..1] and (2t + 8, 2t + 9) in va[mt][2..3].  With kEarly all of them
    // are read into registers here and the slot is released at once; otherwise
    // each is read during the P V product and the slot is released after it.
    uint32_t va[kEarly ? MT : 1][4];
    auto load_v = [&](int mt, uint32_t (&a)[4]) {
      const int t = (mi >> 1) * 8 + rr;
      const int d0 = mt * 16 + (mi & 1) * 8;
      ldmatrix_x4_trans(sv + (d0 / 64) * kSubBytes + swz(t, (d0 % 64) / 8), a[0], a[1], a[2], a[3]);
    };
    if constexpr (kEarly) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) load_v(mt, va[mt]);
      // Invalid tail slots of the last stage hold anything (even NaN): their V
      // values are zeroed here, in registers, so that 0 * NaN cannot reach the
      // accumulator (their scores become -inf below).
      if (n_valid < kStageTokens) {
        const int t2 = 2 * (lane % 4);
        const uint32_t lo = (t2 < n_valid ? 0x0000ffffu : 0u) | (t2 + 1 < n_valid ? 0xffff0000u : 0u);
        const uint32_t hi = (t2 + 8 < n_valid ? 0x0000ffffu : 0u) | (t2 + 9 < n_valid ? 0xffff0000u : 0u);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          va[mt][0] &= lo;
          va[mt][1] &= lo;
          va[mt][2] &= hi;
          va[mt][3] &= hi;
        }
      }
      // Every read of the stage is issued; order them before the refill (an
      // async-proxy write into the same slot) and hand the slot back.
      fence_proxy_async_smem();
      __syncwarp();
      release();
    } else if (n_valid < kStageTokens) {
      // The same masking in shared memory: the invalid V rows become zeros.
      uint4* vz = reinterpret_cast<uint4*>(st + kTileBytes);
      const int nvec = (kStageTokens - n_valid) * 8;  // 128-byte rows, per sub-tile
#pragma unroll
      for (int sb = 0; sb < SUB; ++sb)
        for (int i = lane; i < nvec; i += 32)
          vz[sb * (kSubBytes / 16) + n_valid * 8 + i] = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      __syncwarp();
    }

    const int t0 = lane / 4;
    uint32_t pb[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      if (!live(nt)) {
        pb[nt][0] = pb[nt][1] = 0u;
        continue;
      }
      float x[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = t0 + (j >> 1) * 8;
        bool ok = t < n_valid;
        if (kRows) {
          const int n = nt * 8 + 2 * (lane % 4) + (j & 1);
          ok = ok && n >= r0 && n < r1;
        }
        x[j] = ok ? s[nt][j] * scale_log2 : -INFINITY;
      }
      float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
      for (int off = 4; off < 32; off *= 2) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, off));
      }
      const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
      // O and l are rescaled only when some row's maximum moved (one vote);
      // otherwise every factor is exactly 1.
      if (__any_sync(kFull, (mn0 != m[nt][0]) || (mn1 != m[nt][1]))) {
        float al0 = ex2_approx(m[nt][0] - mn0), al1 = ex2_approx(m[nt][1] - mn1);
        if (kRows) {  // a row with no token so far keeps m = -inf and l = o = 0
          al0 = mn0 == -INFINITY ? 1.f : al0;
          al1 = mn1 == -INFINITY ? 1.f : al1;
        }
        l[nt][0] *= al0;
        l[nt][1] *= al1;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          o[nt][mt][0] *= al0;
          o[nt][mt][1] *= al1;
          o[nt][mt][2] *= al0;
          o[nt][mt][3] *= al1;
        }
        m[nt][0] = mn0;
        m[nt][1] = mn1;
      }
      const float b0 = kRows && mn0 == -INFINITY ? 0.f : mn0;
      const float b1 = kRows && mn1 == -INFINITY ? 0.f : mn1;
      x[0] = ex2_approx(x[0] - b0);
      x[1] = ex2_approx(x[1] - b1);
      x[2] = ex2_approx(x[2] - b0);
      x[3] = ex2_approx(x[3] - b1);
      // Row sums stay per lane (each lane's share of its column); they are added
      // across the column's eight lanes only when the state is read out.
      l[nt][0] += x[0] + x[2];
      l[nt][1] += x[1] + x[3];
      // P (rows t, cols g) -> B fragment of P with k = t, n = g.
      pb[nt][0] = movmatrix_trans(pack_bf16x2(x[0], x[1]));
      pb[nt][1] = movmatrix_trans(pack_bf16x2(x[2], x[3]));
    }

    // O^T += V^T P: one m16n8k16 per (16-dim tile, head tile).
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if constexpr (!kEarly) load_v(mt, va[0]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        if (live(nt)) mma_bf16_16816(o[nt][mt], va[kEarly ? mt : 0], pb[nt][0], pb[nt][1]);
    }
    if constexpr (!kEarly) {
      __syncwarp();
      release();
    }
  }

  // Row sum of column pair (2 (lane % 4), +1) of head tile nt: the per-lane
  // shares added over the eight lanes that hold the column.
  __device__ __forceinline__ float row_sum(int nt, int j) const {
    float x = l[nt][j];
#pragma unroll
    for (int off = 4; off < 32; off *= 2) x += __shfl_xor_sync(kFull, x, off);
    return x;
  }

  __device__ __forceinline__ void store_state(float* dst, int lane) const {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + 2 * (lane % 4);
      const float l0 = row_sum(nt, 0), l1 = row_sum(nt, 1);
      if (lane < 4) {
        dst[g] = m[nt][0];
        dst[g + 1] = m[nt][1];
        dst[GP + g] = l0;
        dst[GP + g + 1] = l1;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int d = mt * 16 + lane / 4;
        dst[2 * GP + g * D + d] = o[nt][mt][0];
        dst[2 * GP + (g + 1) * D + d] = o[nt][mt][1];
        dst[2 * GP + g * D + d + 8] = o[nt][mt][2];
        dst[2 * GP + (g + 1) * D + d + 8] = o[nt][mt][3];
      }
    }
  }

  // Final rows out[g][d] = O^T[d][g] / l[g] for g < G.
  __device__ __forceinline__ void write_out(__nv_bfloat16* out, int G, int lane) const {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + 2 * (lane % 4);
      const float i0 = 1.f / row_sum(nt, 0), i1 = 1.f / row_sum(nt, 1);
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int d = mt * 16 + lane / 4;
        if (g < G) {
          out[g * D + d] = __float2bfloat16_rn(o[nt][mt][0] * i0);
          out[g * D + d + 8] = __float2bfloat16_rn(o[nt][mt][2] * i0);
        }
        if (g + 1 < G) {
          out[(g + 1) * D + d] = __float2bfloat16_rn(o[nt][mt][1] * i1);
          out[(g + 1) * D + d + 8] = __float2bfloat16_rn(o[nt][mt][3] * i1);
        }
      }
    }
  }

  __device__ __forceinline__ void write_partial(float* acc_dst, float2* ml_dst, int G,
                                                int lane) const {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int g = nt * 8 + 2 * (lane % 4);
      const float l0 = row_sum(nt, 0), l1 = row_sum(nt, 1);
      if (lane < 4) {
        if (g < G) ml_dst[g] = make_float2(m[nt][0], l0);
        if (g + 1 < G) ml_dst[g + 1] = make_float2(m[nt][1], l1);
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int d = mt * 16 + lane / 4;
        if (g < G) {
          acc_dst[g * D + d] = o[nt][mt][0];
          acc_dst[g * D + d + 8] = o[nt][mt][2];
        }
        if (g + 1 < G) {
          acc_dst[(g + 1) * D + d] = o[nt][mt][1];
          acc_dst[(g + 1) * D + d + 8] = o[nt][mt][3];
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Fused step: the cache update of token L - 1 of sequence b for KV head kvh,
// after the copy-on-write copy of its block when cow_src[b] >= 0 ("PagedAttention:
// paging the KV cache like an OS pages memory", How it works: a shared block that
// must be modified is copied first).  Only the CTA of the sequence's last
// partition reads that block, so no other CTA needs these writes; the proxy fence
// makes them visible to this CTA's TMA loads.
// ---------------------------------------------------------------------------
template <typename T, int D>
__device__ __forceinline__ void fused_append(const DecodeParams& p, int b, int kvh, int L) {
  const int t = L - 1;
  const int32_t* bt_row = p.block_tables + (size_t)b * p.max_blocks;
  const int dst = bt_row[t / p.bs];
  if (dst < 0 || dst >= p.num_blocks) {
    if (threadIdx.x == 0) flag_error(PKV_DEVERR_BLOCK_ID);
    return;
  }
  constexpr int kVec = D * (int)sizeof(T) / 16;  // 16-byte vectors per head row
  const size_t row_vec = (size_t)p.Hkv * kVec;    // per token row (all heads)
  uint4* kc = reinterpret_cast<uint4*>(p.k_cache_w);
  uint4* vc = reinterpret_cast<uint4*>(p.v_cache_w);
  const int src = p.cow_src != nullptr ? p.cow_src[b] : -1;
  if (src >= p.num_blocks) {
    if (threadIdx.x == 0) flag_error(PKV_DEVERR_COPY);
  } else if (src >= 0 && src != dst) {
    for (int i = threadIdx.x; i < p.bs * kVec; i += blockDim.x) {
      const int r = i / kVec, c = i % kVec;
      const size_t so = ((size_t)src * p.bs + r) * row_vec + (size_t)kvh * kVec + c;
      const size_t d_o = ((size_t)dst * p.bs + r) * row_vec + (size_t)kvh * kVec + c;
      kc[d_o] = kc[so];
      vc[d_o] = vc[so];
    }
    __syncthreads();  // the copy lands before the new token's row overwrites it
  }
  const uint4* kn = reinterpret_cast<const uint4*>(p.k_new);
  const uint4* vn = reinterpret_cast<const uint4*>(p.v_new);
  for (int c = threadIdx.x; c < kVec; c += blockDim.x) {
    const size_t d_o = ((size_t)dst * p.bs + t % p.bs) * row_vec + (size_t)kvh * kVec + c;
    const size_t so = ((size_t)b * p.Hkv + kvh) * kVec + c;
    kc[d_o] = kn[so];
    vc[d_o] = vn[so];
  }
  fence_proxy_async_global();
}

// ---------------------------------------------------------------------------
// The kernel skeleton shared by both consumers.
// ---------------------------------------------------------------------------
template <class C>
struct DecodeSmem {
  static constexpr int kRingBytes = C::kStages * C::kStageBytes;
  static constexpr size_t kBytes =
      1024 /*alignment slack*/ + (size_t)kWarps * kRingBytes + kWarps * C::kStages * 8;
};

// Where a stage's K/V rows are found.
enum : int {
  kLayoutPaged = 0,   // block_size a multiple of 16: a 16-token stage lies in one block
  kLayoutPaged8 = 1,  // block_size 8: a stage spans two blocks (two 8-token boxes)
  kLayoutContig = 2,  // unpaged cache [B][bs][Hkv][D] (bs = the row stride of a sequence):
                      // no block table at all; the control for the paging overhead
};

// Length order, for a few long sequences (B <= kSortedMaxB).  CTAs start in
// the order of their linear block index, and one of them lasts a whole partition,
// so the ones that start last set the end of the launch.  CTA number i therefore
// takes the i-th item of this order: every full partition first (by sequence,
// partition, KV head), then each sequence's last partition from the longest to the
// shortest (an empty sequence counts as a last partition of 0 tokens), so that the
// SMs run out of work together.  Each CTA derives the order from the lengths; it
// returns false when i lies past the last item.
constexpr int kSortedMaxB = 64;

__device__ __forceinline__ bool sorted_item(const DecodeParams& p, int& b, int& part, int& kvh) {
  __shared__ int s_full[kSortedMaxB + 1];  // full partitions of the sequences before b
  __shared__ int s_last[kSortedMaxB];      // tokens of each sequence's last partition
  __shared__ int s_sel;
  const int B = p.B, P = p.part_tokens, Hkv = p.Hkv;
  const int Lcap = min(p.max_blocks * p.bs, p.max_seq_len);
  const int t = threadIdx.x, lane = t % 32;
  const long long i =
      blockIdx.x + (long long)gridDim.x * (blockIdx.y + (long long)gridDim.y * blockIdx.z);
  if (t < 32) {  // lane l: sequences 2l and 2l + 1
    int c[2] = {0, 0};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int x = 2 * lane + h;
      if (x < B) {
        int L = p.seq_lens[x];
        L = L < 0 ? 0 : min(L, Lcap);
        const int n = (L + P - 1) / P;
        c[h] = max(n - 1, 0);
        s_last[x] = L - c[h] * P;
      }
    }
    int inc = c[0] + c[1];  // inclusive scan of the pairs over the lanes
#pragma unroll
    for (int d = 1; d < 32; d *= 2) {
      const int y = __shfl_up_sync(kFull, inc, d);
      if (lane >= d) inc += y;
    }
    const int before = inc - c[0] - c[1];
    if (2 * lane < B) s_full[2 * lane + 1] = before + c[0];
    if (2 * lane + 1 < B) s_full[2 * lane + 2] = before + c[0] + c[1];
    if (lane == 0) s_full[0] = 0;
  }
  __syncthreads();
  const long long f = i / Hkv;
  kvh = (int)(i % Hkv);
  const int F = s_full[B];
  if (f < F) {
    int lo = 0, hi = B;  // s_full[lo] <= f < s_full[hi]
    while (hi - lo > 1) {
      const int mid = (lo + hi) / 2;
      if (s_full[mid] <= f) lo = mid;
      else hi = mid;
    }
    b = lo;
    part = (int)(f - s_full[lo]);
    return true;
  }
  const long long j = f - F;
  if (j >= B) return false;
  if (t < B) {
    const int mine = s_last[t];
    int rank = 0;
    for (int x = 0; x < B; ++x) {
      const int o = s_last[x];
      rank += (o > mine) || (o == mine && x < t);
    }
    if (rank == j) s_sel = t;
  }
  __syncthreads();
  b = s_sel;
  part = s_full[b + 1] - s_full[b];  // its full partitions come before the last one
  return true;
}

template <class C, typename T, int D, int LAYOUT = kLayoutPaged>
__global__ void __launch_bounds__(kWarps * 32)
    paged_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV) {
  launch_overlap_entry();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int kRing = DecodeSmem<C>::kRingBytes;
  static_assert(kRing >= (2 * C::GP + C::GP * D) * 4, "state does not fit in the ring");
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kRing);
  __shared__ float s_M[16], s_den[16];
  __shared__ int s_last;

  int kvh = blockIdx.x, part = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G;
  const int P = p.part_tokens;

  // After a pipeline timeout anywhere, later CTAs stop at once instead of waiting too.
  if (cta_timed_out()) return;
  if (p.sorted && !sorted_item(p, b, part, kvh)) return;
  int L = p.seq_lens[b];
  const int Lcap = min(p.max_blocks * p.bs, p.max_seq_len);
  if (L < 0 || L > Lcap) {
    if (threadIdx.x == 0 && part == 0 && kvh == 0) flag_error(PKV_DEVERR_SEQLEN);
    L = L < 0 ? 0 : Lcap;
  }
  const int nparts = (L + P - 1) / P;
  T* out = reinterpret_cast<T*>(p.out) + ((size_t)b * p.Hq + (size_t)kvh * G) * D;
  if (L == 0) {
    if (part == 0)
      for (int i = threadIdx.x; i < G * D; i += blockDim.x) out[i] = to_out<T>(0.f);
    return;
  }
  if (part >= nparts) return;
  if (p.k_new != nullptr && part == nparts - 1) {
    fused_append<T, D>(p, b, kvh, L);
    __syncthreads();
  }

  const int t_begin = part * P;
  const int t_end = min(L, t_begin + P);
  const int n_st = (t_end - t_begin + kStageTokens - 1) / kStageTokens;
  const int n_w = n_st > warp ? (n_st - warp + kWarps - 1) / kWarps : 0;

  uint8_t* ring = smem + warp * kRing;
  uint64_t* wbar = bars + warp * C::kStages;
  if (lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
#pragma unroll
    for (int s = 0; s < C::kStages; ++s) mbar_init(&wbar[s], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const uint64_t pol = l2_policy_evict_first();
  const int32_t* bt_row = p.block_tables + (size_t)b * p.max_blocks;
  // Physical id of the block holding tokens t0 + 8 * half .. of stage k (half 1 only
  // with 8-token blocks, and only when the partition has tokens there).
  auto stage_id = [&](int k, int half) -> int {
    const int t0 = t_begin + (warp + kWarps * k) * kStageTokens + 8 * half;
    if constexpr (LAYOUT == kLayoutContig) return b;
    if (half && t0 >= t_end) return 0;
    return bt_row[t0 / p.bs];
  };
  // Physical ids of this warp's stages win_base .. win_base+63 (one per lane, two
  // windows; with 8-token blocks a second pair for the stages' second halves).
  constexpr bool kTwo = LAYOUT == kLayoutPaged8;
  int win_base = 0;
  int win0 = lane < n_w ? stage_id(lane, 0) : -1;
  int win1 = 32 + lane < n_w ? stage_id(32 + lane, 0) : -1;
  int win0b = kTwo && lane < n_w ? stage_id(lane, 1) : -1;
  int win1b = kTwo && 32 + lane < n_w ? stage_id(32 + lane, 1) : -1;

  auto issue = [&](int k) {
    if (k - win_base >= 32) {
      win0 = win1;
      win_base += 32;
      win1 = win_base + 32 + lane < n_w ? stage_id(win_base + 32 + lane, 0) : -1;
      if constexpr (kTwo) {
        win0b = win1b;
        win1b = win_base + 32 + lane < n_w ? stage_id(win_base + 32 + lane, 1) : -1;
      }
    }
    // After the rotation above, k - win_base < 32: read win0 only.  (Naming win1
    // here would make the shuffle wait for the window load just issued.)
    const int id = __shfl_sync(kFull, win0, k - win_base);
    const int id_b = kTwo ? __shfl_sync(kFull, win0b, k - win_base) : 0;
    if (lane == 0) {
      const int s = k % C::kStages;
      const int t0 = t_begin + (warp + kWarps * k) * kStageTokens;
      const int oob = p.num_blocks * p.bs;  // entirely out of bounds: TMA fills zeros
      auto row_of = [&](int id_, int t) -> int {
        if (id_ < 0 || id_ >= p.num_blocks) {
          flag_error(PKV_DEVERR_BLOCK_ID);
          return oob;
        }
        return id_ * p.bs + t % p.bs;
      };
      mbar_arrive_expect_tx(&wbar[s], C::kStageBytes);
      if constexpr (kTwo) {
        // No tokens in the second half: a zero box, not a table read.
        const int row1 = t0 + 8 < t_end ? row_of(id_b, t0 + 8) : oob;
        C::load_stage_halves(ring + s * C::kStageBytes, &tmK, &tmV, &wbar[s], kvh,
                             row_of(id, t0), row1, pol);
      } else {
        C::load_stage(ring + s * C::kStageBytes, &tmK, &tmV, &wbar[s], kvh, row_of(id, t0), pol);
      }
    }
  };

  const int n_pro = n_w < C::kStages ? n_w : C::kStages;
  for (int k = 0; k < n_pro; ++k) issue(k);

  C c;
  c.init(p, b, kvh, lane);

  for (int k = 0; k < n_w; ++k) {
    const int s = k % C::kStages;
    const uint32_t parity = (uint32_t)((k / C::kStages) & 1);
    const bool ok = mbar_wait_bounded(&wbar[s], parity);
    if (__any_sync(kFull, !ok)) {
      // Give up: flag it, wait (bounded) for the other loads in flight, stop.
      if (lane == 0) flag_error(PKV_DEVERR_TIMEOUT);
      for (int j = k; j < n_w && j < k + C::kStages; ++j)
        mbar_wait_bounded(&wbar[j % C::kStages], (uint32_t)((j / C::kStages) & 1));
      break;
    }
    const int t0 = t_begin + (warp + kWarps * k) * kStageTokens;
    const int n_valid = min(kStageTokens, t_end - t0);
    c.consume(ring + s * C::kStageBytes, n_valid, lane, [&] {
      if (k + C::kStages < n_w) issue(k + C::kStages);
    });
  }

  // Merge the warps' states (each in its own, now idle, ring).
  c.store_state(reinterpret_cast<float*>(ring), lane);
  __syncthreads();
  constexpr int GP = C::GP;
  const bool split = nparts > 1;
  const size_t unit = (size_t)b * p.Hkv + kvh;
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      M = fmaxf(M, reinterpret_cast<const float*>(smem + w * kRing)[g]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* st = reinterpret_cast<const float*>(smem + w * kRing);
      const float f = exp2f(st[g] - M);
      num = fmaf(f, st[2 * GP + g * D + d], num);
      den = fmaf(f, st[GP + g], den);
    }
    if (!split) {
      out[idx] = to_out<T>(num / den);
    } else {
      const size_t u = (unit * p.max_parts + part) * G + g;
      p.ws_acc[u * D + d] = num;
      if (d == 0) p.ws_ml[u] = make_float2(M, den);
    }
  }
  if (!split) return;

  // Partition merge: the last CTA of this (b, kvh) to finish does it.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prev = atomicAdd(&p.ws_count[unit], 1u);
    s_last = (prev == (uint32_t)(nparts - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const size_t base = unit * p.max_parts * G;
  // Each partial's weight exp2(m_q - M) / den, formed once per (partition, head)
  // into the shared memory the stages no longer use; then every thread sums
  // 4-float chunks of the output with kU partials' loads in flight.  (A loop over
  // the partials one at a time was bound by L2 latency: 17-45 us per merge on the
  // long-context workload, at the very end of the launch.)
  constexpr int kU = 16;
  float* s_w = reinterpret_cast<float*>(smem);  // [partition][head]
  const bool fast = nparts * G <= kWarps * kRing / (int)sizeof(float) && D % 4 == 0;
  for (int g = warp; g < G; g += kWarps) {
    float M = -INFINITY, den = 0.f;
    if (nparts <= 32) {  // one (max, sum) a lane, read once
      const float2 ml = lane < nparts ? __ldcg(&p.ws_ml[base + (size_t)lane * G + g])
                                      : make_float2(-INFINITY, 0.f);
      M = ml.x;
#pragma unroll
      for (int off = 16; off >= 1; off /= 2) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
      const float e = lane < nparts ? exp2f(ml.x - M) : 0.f;
      den = e * ml.y;
#pragma unroll
      for (int off = 16; off >= 1; off /= 2) den += __shfl_xor_sync(kFull, den, off);
      if (fast && lane < nparts) s_w[lane * G + g] = e / den;
    } else {
      for (int q = lane; q < nparts; q += 32) M = fmaxf(M, __ldcg(&p.ws_ml[base + (size_t)q * G + g]).x);
#pragma unroll
      for (int off = 16; off >= 1; off /= 2) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
      for (int q = lane; q < nparts; q += 32) {
        const float2 ml = __ldcg(&p.ws_ml[base + (size_t)q * G + g]);
        den += exp2f(ml.x - M) * ml.y;
      }
#pragma unroll
      for (int off = 16; off >= 1; off /= 2) den += __shfl_xor_sync(kFull, den, off);
      if (fast) {
        const float inv = 1.f / den;
        for (int q = lane; q < nparts; q += 32)
          s_w[q * G + g] = exp2f(__ldcg(&p.ws_ml[base + (size_t)q * G + g]).x - M) * inv;
      }
    }
    if (lane == 0) {
      s_M[g] = M;
      s_den[g] = den;
    }
  }
  __syncthreads();
  if (fast) {
    for (int c = threadIdx.x; c < G * D / 4; c += blockDim.x) {
      const int g = c / (D / 4), d4 = c % (D / 4);
      const float4* src = reinterpret_cast<const float4*>(p.ws_acc + (base + g) * D) + d4;
      const size_t stride = (size_t)G * D / 4;  // float4s from one partition's row g to the next
      float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
      int q = 0;
      for (; q + kU <= nparts; q += kU) {
        float4 v[kU];
#pragma unroll
        for (int k = 0; k < kU; ++k) v[k] = __ldcg(src + (size_t)(q + k) * stride);
#pragma unroll
        for (int k = 0; k < kU; ++k) {
          const float w = s_w[(q + k) * G + g];
          a.x = fmaf(w, v[k].x, a.x);
          a.y = fmaf(w, v[k].y, a.y);
          a.z = fmaf(w, v[k].z, a.z);
          a.w = fmaf(w, v[k].w, a.w);
        }
      }
      for (; q < nparts; ++q) {
        const float4 v = __ldcg(src + (size_t)q * stride);
        const float w = s_w[q * G + g];
        a.x = fmaf(w, v.x, a.x);
        a.y = fmaf(w, v.y, a.y);
        a.z = fmaf(w, v.z, a.z);
        a.w = fmaf(w, v.w, a.w);
      }
      T* o = out + g * D + 4 * d4;
      o[0] = to_out<T>(a.x);
      o[1] = to_out<T>(a.y);
      o[2] = to_out<T>(a.z);
      o[3] = to_out<T>(a.w);
    }
    if (threadIdx.x == 0) p.ws_count[unit] = 0u;
    return;
  }
  for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
    const int g = idx / D, d = idx % D;
    const float M = s_M[g];
    float num = 0.f;
    for (int q = 0; q < nparts; ++q) {
      const size_t u = base + (size_t)q * G + g;
      num = fmaf(exp2f(__ldcg(&p.ws_ml[u]).x - M), __ldcg(&p.ws_acc[u * D + d]), num);
    }
    out[idx] = to_out<T>(num / s_den[g]);
  }
  if (threadIdx.x == 0) p.ws_count[unit] = 0u;
}

}  // namespace pkv
