// Work-balanced persistent variant of the paged decode (sm_100a).
//
// Same arithmetic as paged_decode_kernel (see pkv_decode.cuh); what changes is
// how the work is cut.  For each KV head h, the sequences' 16-token stages are
// laid end to end into one stream of S_h = sum_b ceil(L_b / 16) stages (the
// same length for every head).  Each head's stream is cut into NG equal
// contiguous ranges; warp ("worker") g*Hkv + h takes range g of head h.  So:
//  * every worker moves the same number of K/V bytes (to within one stage):
//    no idle CTAs for short sequences, no tail of long ones;
//  * the Hkv workers of one group walk the same sequences and stages at the
//    same pace, reading the Hkv head slices of the same physical blocks
//    together, so each block's K/V rows are read from DRAM as a whole;
//  * each worker fills its TMA pipeline once and keeps it full across
//    sequence boundaries (the block ids of its next 32..64 stages are kept in
//    registers, and q of its next sequence is prefetched into L2).
//
// A unit (b, h) that lies inside one range is finished by that worker.  A unit
// cut by range boundaries leaves one partial (max, sum, weighted V) per group
// that touched it, in slot h*(B + NG) + b + g: along the staircase of (b, g)
// pairs of one head that sum strictly increases, so slots never collide.  The
// worker whose atomic ticket comes last merges the unit (no spinning).
#pragma once

#include "pkv_decode.cuh"

namespace pkv {

constexpr int kBalancedMaxB = 2048;        // per-sequence prefix kept in smem
constexpr int kBalancedMaxCtas = 2 * 148;  // 2 resident CTAs per SM
constexpr int kBalancedMaxWorkers = kBalancedMaxCtas * kWarps;

// Partial slots: Hkv * (B + NG) with NG <= max(1, workers / Hkv).
__host__ __device__ constexpr size_t balanced_slots(size_t B, size_t Hkv) {
  return Hkv * B + (Hkv > (size_t)kBalancedMaxWorkers ? Hkv : (size_t)kBalancedMaxWorkers);
}

template <class C>
struct BalancedSmem {
  static constexpr size_t kBase = DecodeSmem<C>::kBytes;  // rings + barriers + alignment slack
  static constexpr size_t bytes(int B) { return kBase + (size_t)(B + 1) * sizeof(int); }
};

__device__ __forceinline__ int clamp_len(int L, int Lcap, bool report) {
  if (L < 0 || L > Lcap) {
    if (report) flag_error(PKV_DEVERR_SEQLEN);
    return L < 0 ? 0 : Lcap;
  }
  return L;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

template <class C, typename T, int D>
__global__ void __launch_bounds__(kWarps * 32)
    paged_decode_balanced_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                                 const __grid_constant__ CUtensorMap tmV) {
  launch_overlap_entry();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  constexpr int kRing = DecodeSmem<C>::kRingBytes;
  constexpr int NS = C::kStages;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kRing);
  int* s_pre = reinterpret_cast<int*>(bars + kWarps * NS);  // [B + 1]
  __shared__ int s_warp_tot[kWarps];

  if (cta_timed_out()) return;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int B = p.B, Hkv = p.Hkv, G = p.G;
  const int Lcap = min(p.max_blocks * p.bs, p.max_seq_len);
  const bool report = blockIdx.x == 0;

  // 1) Per-head stage prefix over sequences: s_pre[b] = sum_{b' < b} ceil(L_b' / 16).
  const int chunk = (B + blockDim.x - 1) / blockDim.x;
  const int b0 = threadIdx.x * chunk;
  int local = 0;
  for (int i = 0; i < chunk; ++i) {
    const int b = b0 + i;
    if (b < B) local += (clamp_len(p.seq_lens[b], Lcap, report) + kStageTokens - 1) / kStageTokens;
  }
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off *= 2) {
    const int v = __shfl_up_sync(kFull, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) s_warp_tot[warp] = incl;
  __syncthreads();
  int ex = incl - local;
  int total = 0;
#pragma unroll
  for (int w2 = 0; w2 < kWarps; ++w2) {
    if (w2 < warp) ex += s_warp_tot[w2];
    total += s_warp_tot[w2];
  }
  for (int i = 0; i < chunk; ++i) {
    const int b = b0 + i;
    if (b < B) {
      s_pre[b] = ex;
      ex += (clamp_len(p.seq_lens[b], Lcap, false) + kStageTokens - 1) / kStageTokens;
    }
  }
  if (threadIdx.x == 0) s_pre[B] = total;
  __syncthreads();

  // Empty sequences produce zero rows (no worker range touches them).
  T* out_all = reinterpret_cast<T*>(p.out);
  for (int b = blockIdx.x; b < B; b += gridDim.x)
    if (s_pre[b + 1] == s_pre[b])
      for (int i = threadIdx.x; i < p.Hq * D; i += blockDim.x)
        out_all[(size_t)b * p.Hq * D + i] = to_out<T>(0.f);

  // 2) Workers.  NG groups per head, at most one stage-range each way: NG <= S
  //    keeps every range non-empty, so a unit's pieces are exactly the groups
  //    group_of(first) .. group_of(last), which the merge ticket counts.
  //    Virtual worker v = g*Hkv + h runs on warp v mod (warps in the grid).
  const int S = s_pre[B];
  if (S == 0) return;  // no CTA-wide barrier follows
  const int Wk = gridDim.x * kWarps;
  const int NG = max(1, min(Wk / Hkv, S));
  const int V = NG * Hkv;
  const int w = blockIdx.x * kWarps + warp;
  if (w >= V) return;
  auto group_of = [&](int pos) -> int { return (int)(((int64_t)(pos + 1) * NG + S - 1) / S) - 1; };
  auto find_b = [&](int pos) -> int {  // s_pre[b] <= pos < s_pre[b + 1]
    int lo = 0, hi = B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_pre[mid] <= pos) lo = mid; else hi = mid;
    }
    return lo;
  };
  auto next_b = [&](int b) -> int {  // next sequence with at least one token (or B)
    do { ++b; } while (b < B && s_pre[b + 1] == s_pre[b]);
    return b;
  };
  const size_t q_bytes = (size_t)G * D * sizeof(T);
  auto prefetch_unit = [&](int b, int h) {  // q rows and length of unit (b, h) into L2
    if (b >= B) return;
    const char* qrow = reinterpret_cast<const char*>(p.q) + ((size_t)b * p.Hq + (size_t)h * G) * D * sizeof(T);
    for (size_t off = (size_t)lane * 128; off < q_bytes; off += 32 * 128) prefetch_l2(qrow + off);
    if (lane == 0) prefetch_l2(p.seq_lens + b);
  };

  uint8_t* ring = smem + warp * kRing;
  uint64_t* wbar = bars + warp * NS;
  if (lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
#pragma unroll
    for (int s = 0; s < NS; ++s) mbar_init(&wbar[s], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_policy_evict_first();
  uint32_t kbase = 0;  // stages this warp has consumed: ring slot and phase continue across v

  for (int v = w; v < V; v += Wk) {
    const int g = v / Hkv, h = v % Hkv;
    const int p_begin = (int)((int64_t)g * S / NG);
    const int p_end = (int)((int64_t)(g + 1) * S / NG);
    const int n = p_end - p_begin;

    // Raw block id and in-block row offset of stage p_begin + k (32 stages per lane window).
    auto locate = [&](int k, int& id, int& sub) {
      id = -1;
      sub = 0;
      if (k >= n) return;
      const int pos = p_begin + k;
      const int b = find_b(pos);
      const int t0 = (pos - s_pre[b]) * kStageTokens;
      id = p.block_tables[(size_t)b * p.max_blocks + t0 / p.bs];
      sub = t0 % p.bs;
    };
    int win_base = 0, id0, sub0, id1, sub1;
    locate(lane, id0, sub0);
    locate(32 + lane, id1, sub1);
    auto issue = [&](int k) {
      if (k - win_base >= 32) {
        id0 = id1;
        sub0 = sub1;
        win_base += 32;
        locate(win_base + 32 + lane, id1, sub1);  // consumed 32 stages from now
      }
      // After the rotation above, k - win_base < 32: read window 0 only.  (Naming
      // window 1 here would make the shuffle wait for the load just issued.)
      const int id = __shfl_sync(kFull, id0, k - win_base);
      const int sub = __shfl_sync(kFull, sub0, k - win_base);
      if (lane == 0) {
        int row;
        if (id < 0 || id >= p.num_blocks) {
          flag_error(PKV_DEVERR_BLOCK_ID);
          row = p.num_blocks * p.bs;  // entirely out of bounds: TMA fills zeros
        } else {
          row = id * p.bs + sub;
        }
        const uint32_t r = (kbase + k) % NS;
        mbar_arrive_expect_tx(&wbar[r], C::kStageBytes);
        C::load_stage(ring + r * C::kStageBytes, &tmK, &tmV, &wbar[r], h, row, pol);
      }
    };
    const int n_pro = n < NS ? n : NS;
    for (int k = 0; k < n_pro; ++k) issue(k);

    // 3) Consume the range sequence by sequence.
    int pos = p_begin;
    int b = find_b(pos);
    int st = pos - s_pre[b];
    int nst = s_pre[b + 1] - s_pre[b];
    int L = clamp_len(p.seq_lens[b], Lcap, false);
    C c;
    c.init(p, b, h, lane);
    prefetch_unit(next_b(b), h);
    for (int k = 0; k < n; ++k) {
      const uint32_t kk = kbase + k;
      const bool ok = mbar_wait_bounded(&wbar[kk % NS], (kk / NS) & 1u);
      if (__any_sync(kFull, !ok)) {
        if (lane == 0) flag_error(PKV_DEVERR_TIMEOUT);
        for (int j = k; j < n && j < k + NS; ++j)
          mbar_wait_bounded(&wbar[(kbase + j) % NS], ((kbase + j) / NS) & 1u);
        return;
      }
      c.consume(ring + (kk % NS) * C::kStageBytes, min(kStageTokens, L - st * kStageTokens), lane,
                [&] {
                  if (k + NS < n) issue(k + NS);
                });
      ++st;
      ++pos;
      if (st < nst && pos < p_end) continue;

      // This worker's piece of unit (b, h) is done.
      const int u = b * Hkv + h;
      const int gf = group_of(s_pre[b]), gl = group_of(s_pre[b + 1] - 1);
      T* orow = out_all + ((size_t)b * p.Hq + (size_t)h * G) * D;
      if (gf == gl) {
        c.write_out(orow, G, lane);
      } else {
        const size_t head_base = (size_t)h * (B + NG);
        const size_t slot = head_base + b + g;
        c.write_partial(p.ws_acc + slot * G * D, p.ws_ml + slot * G, G, lane);
        __threadfence();
        __syncwarp();
        uint32_t last = 0;
        if (lane == 0) last = atomicAdd(&p.ws_count[u], 1u) == (uint32_t)(gl - gf);
        last = __shfl_sync(kFull, last, 0);
        if (last) {
          __threadfence();
          bool continue_after_merge = false;  // the fast merge below did the unit
          const size_t base = head_base + b + gf;
          const int nseg = gl - gf + 1;
          if (nseg <= 32 && D == 128) {
            // Lane q holds piece q's weight exp2(m_q - M) / den of the row; then lane
            // l sums dims 4l .. 4l + 3 over the pieces, kU pieces' loads in flight.
            // (One piece at a time was bound by L2 latency.)
            constexpr int kU = 8;
            for (int gg = 0; gg < G; ++gg) {
              const float2 ml = lane < nseg ? __ldcg(&p.ws_ml[(base + lane) * G + gg])
                                            : make_float2(-INFINITY, 0.f);
              float M = ml.x;
#pragma unroll
              for (int off = 16; off >= 1; off /= 2) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
              const float e = lane < nseg ? exp2f(ml.x - M) : 0.f;
              float den = e * ml.y;
#pragma unroll
              for (int off = 16; off >= 1; off /= 2) den += __shfl_xor_sync(kFull, den, off);
              const float w = e / den;
              const float4* src = reinterpret_cast<const float4*>(p.ws_acc + (base * G + gg) * D) + lane;
              const size_t stride = (size_t)G * D / 4;  // float4s from one piece to the next
              float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
              for (int q0 = 0; q0 < nseg; q0 += kU) {
                float4 v[kU];
#pragma unroll
                for (int k = 0; k < kU; ++k)
                  v[k] = q0 + k < nseg ? __ldcg(src + (size_t)(q0 + k) * stride)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int k = 0; k < kU; ++k) {
                  const float wq = __shfl_sync(kFull, w, (q0 + k) & 31);
                  a.x = fmaf(wq, v[k].x, a.x);
                  a.y = fmaf(wq, v[k].y, a.y);
                  a.z = fmaf(wq, v[k].z, a.z);
                  a.w = fmaf(wq, v[k].w, a.w);
                }
              }
              T* o = orow + gg * D + 4 * lane;
              o[0] = to_out<T>(a.x);
              o[1] = to_out<T>(a.y);
              o[2] = to_out<T>(a.z);
              o[3] = to_out<T>(a.w);
            }
            if (lane == 0) p.ws_count[u] = 0u;
            continue_after_merge = true;
          }
          for (int gg = 0; gg < G && !continue_after_merge; ++gg) {
            float M = -INFINITY;
            for (int q = lane; q < nseg; q += 32) M = fmaxf(M, __ldcg(&p.ws_ml[(base + q) * G + gg]).x);
#pragma unroll
            for (int off = 16; off >= 1; off /= 2) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
            float den = 0.f;
            for (int q = lane; q < nseg; q += 32) {
              const float2 ml = __ldcg(&p.ws_ml[(base + q) * G + gg]);
              den += exp2f(ml.x - M) * ml.y;
            }
#pragma unroll
            for (int off = 16; off >= 1; off /= 2) den += __shfl_xor_sync(kFull, den, off);
            for (int d = lane; d < D; d += 32) {
              float num = 0.f;
              for (int q = 0; q < nseg; ++q) {
                const float mq = __ldcg(&p.ws_ml[(base + q) * G + gg]).x;
                num = fmaf(exp2f(mq - M), __ldcg(&p.ws_acc[((base + q) * G + gg) * D + d]), num);
              }
              orow[gg * D + d] = to_out<T>(num / den);
            }
          }
          if (!continue_after_merge && lane == 0) p.ws_count[u] = 0u;
        }
      }
      if (pos >= p_end) break;
      b = next_b(b);  // pos < p_end, so a later sequence with tokens exists
      st = 0;
      nst = s_pre[b + 1] - s_pre[b];
      L = clamp_len(p.seq_lens[b], Lcap, false);
      c.init(p, b, h, lane);
      prefetch_unit(next_b(b), h);
    }
    kbase += (uint32_t)n;
  }
}

}  // namespace pkv
