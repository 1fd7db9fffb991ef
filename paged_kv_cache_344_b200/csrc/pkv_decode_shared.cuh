// Shared-prefix decode (sm_100a): blocks shared by several sequences are read
// once for all of them.
//
// Physical blocks may be shared between sequences -- decode branches of one
// request, parallel samples, a common prompt -- through identical block-table
// entries ("PagedAttention: paging the KV cache like an OS pages memory", How
// it works).  The plain decode reads a shared block once per sequence.  Here
// the caller lists groups of consecutive sequences whose first prefix_len
// tokens sit in the same physical blocks, and the work is cut into
//  * prefix pieces: (group, member chunk, prefix partition, KV head).  One CTA
//    reads the partition's K/V once and scores it against the queries of up
//    to 16 / G members at once: their G heads each stack into the N dimension
//    of the tensor-core MMA (16 rows);
//  * own pieces: (sequence, own partition, KV head) over the tokens after the
//    prefix, exactly as in the plain decode.
// Every piece leaves a partial (max, sum, weighted V) per (sequence, head); the
// piece whose atomic ticket comes last for a (sequence, KV head) merges them
// with a log-sum-exp rescale.  The result is the same softmax attention.
//
// Robustness: the prefix used for a group is shortened to one token less than
// the shortest member and rounded down to whole blocks; a prefix piece checks that
// every member's table entries for its blocks equal the first member's.  A
// mismatch, or group offsets that do not cover the batch, flags
// PKV_DEVERR_PREFIX (results are then unreliable; memory stays in bounds).
#pragma once

#include "pkv_decode.cuh"

namespace pkv {

struct SharedParams {
  DecodeParams d;                // out, q, tables, lengths, shapes, scale
  const int32_t* group_offsets;  // [n_groups + 1]: group g = sequences off[g] .. off[g+1]-1
  const int32_t* prefix_lens;    // [n_groups]
  float* ws_acc;                 // [B*Hkv][slots][G][D]
  float2* ws_ml;                 // [B*Hkv][slots][G]
  uint32_t* ws_count;            // [B*Hkv]
  int n_groups;
  int chunks;     // member chunks per group (ceil(max group size / mc))
  int mc;         // members per prefix piece: max(1, 16 / G)
  int max_pp;     // prefix partitions per group (upper bound)
  int max_op;     // own partitions per sequence (upper bound)
  int max_group;  // largest group size (upper bound)
  int P;          // partition length (tokens, multiple of 16)
  int n_prefix_items;
};

__device__ __forceinline__ int shared_len(const DecodeParams& d, int b) {
  const int cap = min(d.max_blocks * d.bs, d.max_seq_len);
  const int L = d.seq_lens[b];
  return L < 0 ? 0 : (L > cap ? cap : L);
}

// Prefix actually shared by group g: short of every member's newest token, and
// whole blocks (block_size is a multiple of the 16-token stage).  So no block of
// the prefix is the one that receives a member's new token, which a fused step
// rewrites (copy-on-write copy and the new row) while prefix pieces read.
__device__ __forceinline__ int group_prefix(const SharedParams& s, int g, int lo, int hi) {
  int plen = s.prefix_lens[g];
  int minL = 0x7fffffff;
  for (int b = lo; b < hi; ++b) minL = min(minL, shared_len(s.d, b) - 1);
  if (hi <= lo) minL = 0;
  plen = max(0, min(plen, minL));
  return plen / s.d.bs * s.d.bs;
}

// Group offset g clamped into [0, B]: offsets are caller data, and no value of
// theirs may lead outside the batch.
__device__ __forceinline__ int group_off(const SharedParams& s, int g) {
  const int x = s.group_offsets[g];
  return x < 0 ? 0 : (x > s.d.B ? s.d.B : x);
}

__device__ __forceinline__ void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ int ceil_div_i(int a, int b) { return (a + b - 1) / b; }

// What one CTA of the shared-prefix grid does.
struct SharedItem {
  bool valid;
  bool prefix;
  int kvh;
  int b0;          // first sequence of the rows (prefix: first member of the chunk)
  int members;     // rows are members x G (own pieces: 1)
  int table_b;     // sequence whose table row gives the block ids
  int t_begin, t_end;
  int slot;        // partial slot of this piece for each of its sequences
  int plen;        // shared prefix of the group (tokens)
  int npp;         // prefix partitions of the group
};

__device__ __forceinline__ SharedItem decode_shared_item(const SharedParams& s, int x) {
  SharedItem it;
  it.valid = false;
  it.prefix = x < s.n_prefix_items;
  const int Hkv = s.d.Hkv;
  it.kvh = x % Hkv;
  int rest = x / Hkv;
  if (it.prefix) {
    const int pp = rest % s.max_pp;
    rest /= s.max_pp;
    const int c = rest % s.chunks;
    const int g = rest / s.chunks;
    const int lo = group_off(s, g), hi = max(lo, group_off(s, g + 1));
    it.b0 = lo + c * s.mc;
    it.members = min(s.mc, hi - it.b0);
    if (it.members <= 0) return it;
    it.plen = group_prefix(s, g, lo, hi);
    it.npp = ceil_div_i(it.plen, s.P);
    if (pp >= it.npp) return it;
    it.table_b = lo;
    it.t_begin = pp * s.P;
    it.t_end = min(it.plen, it.t_begin + s.P);
    it.slot = pp;
  } else {
    // Own pieces are enumerated per group, (g, member j, own partition, KV head),
    // so a piece finds its sequence from two offsets instead of a search.
    rest = (x - s.n_prefix_items) / Hkv;
    const int op = rest % s.max_op;
    rest /= s.max_op;
    const int j = rest % s.max_group;
    const int g = rest / s.max_group;
    const int lo = group_off(s, g), hi = max(lo, group_off(s, g + 1));
    const int b = lo + j;
    if (b >= hi) return it;
    it.plen = group_prefix(s, g, lo, hi);
    it.npp = ceil_div_i(it.plen, s.P);
    const int L = shared_len(s.d, b);
    it.b0 = b;
    it.members = 1;
    it.table_b = b;
    it.t_begin = it.plen + op * s.P;
    it.t_end = min(L, it.t_begin + s.P);
    // An empty sequence still needs its zero rows: own partition 0 writes them.
    if (it.t_begin >= it.t_end && !(L == 0 && op == 0)) return it;
    it.slot = s.max_pp + op;
  }
  it.valid = true;
  return it;
}

// Pieces that contribute to (b, kvh): the group's prefix partitions + own ones.
__device__ __forceinline__ int pieces_of(const SharedParams& s, int b, int plen, int npp) {
  const int L = shared_len(s.d, b);
  return npp + ceil_div_i(max(L - plen, 0), s.P);
}

// One piece, run with consumer C (16 query rows for prefix pieces, the
// smallest that holds G rows for own pieces).
template <class C, int D>
__device__ __forceinline__ void shared_piece(const SharedParams& s, const SharedItem& it,
                                             uint8_t* smem, const CUtensorMap& tmK,
                                             const CUtensorMap& tmV, float* s_M, float* s_den,
                                             int& s_last) {
  using T = __nv_bfloat16;
  constexpr int kRing = DecodeSmem<C>::kRingBytes;
  static_assert(kRing >= (2 * C::GP + C::GP * D) * 4, "state does not fit in the ring");
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWarps * kRing);
  const DecodeParams& p = s.d;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G, kvh = it.kvh, Hkv = p.Hkv;
  T* out = reinterpret_cast<T*>(p.out);
  if (it.t_begin >= it.t_end) {  // an empty sequence: zero rows
    T* o = out + ((size_t)it.b0 * p.Hq + (size_t)kvh * G) * D;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) o[i] = __float2bfloat16_rn(0.f);
    return;
  }
  if (!it.prefix && p.k_new != nullptr && it.t_end == shared_len(p, it.b0)) {
    // Fused step: this own piece holds the sequence's new token (never inside the
    // shared prefix), so it alone reads that token's block.
    fused_append<T, D>(p, it.b0, kvh, it.t_end);
    __syncthreads();
  }
  const int32_t* bt_row = p.block_tables + (size_t)it.table_b * p.max_blocks;
  // Start the q rows and this piece's table entries on their way to L2 now.
  {
    const char* qrow = reinterpret_cast<const char*>(p.q) +
                       ((size_t)it.b0 * p.Hq + (size_t)kvh * G) * D * sizeof(T);
    const int lines = G * D * (int)sizeof(T) / 128;  // 128-byte lines of one member's rows
    if ((int)threadIdx.x < it.members * lines) {
      const int i = threadIdx.x / lines, line = threadIdx.x % lines;
      prefetch_l2_line(qrow + (size_t)i * p.Hq * D * sizeof(T) + (size_t)line * 128);
    }
    const int tb0 = it.t_begin / p.bs, tb1 = (it.t_end - 1) / p.bs;
    for (int j = tb0 + 32 * (int)threadIdx.x; j <= tb1; j += 32 * blockDim.x) prefetch_l2_line(bt_row + j);
  }
  if (it.prefix) {  // every member must hold the same physical blocks for the prefix
    const int j0 = it.t_begin / p.bs, j1 = (it.t_end - 1) / p.bs;
    const int nj = j1 - j0 + 1;
    for (int x = threadIdx.x; x < nj * it.members; x += blockDim.x) {
      const int j = j0 + x % nj, b = it.b0 + x / nj;
      if (p.block_tables[(size_t)b * p.max_blocks + j] != bt_row[j]) flag_error(PKV_DEVERR_PREFIX);
    }
  }

  const int t_begin = it.t_begin, t_end = it.t_end;
  const int n_st = (t_end - t_begin + kStageTokens - 1) / kStageTokens;
  const int n_w = n_st > warp ? (n_st - warp + kWarps - 1) / kWarps : 0;
  uint8_t* ring = smem + warp * kRing;
  uint64_t* wbar = bars + warp * C::kStages;
  if (lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
#pragma unroll
    for (int st = 0; st < C::kStages; ++st) mbar_init(&wbar[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_policy_evict_first();
  auto stage_id = [&](int k) -> int {
    return bt_row[(t_begin + (warp + kWarps * k) * kStageTokens) / p.bs];
  };
  int win_base = 0;
  int win0 = lane < n_w ? stage_id(lane) : -1;
  int win1 = 32 + lane < n_w ? stage_id(32 + lane) : -1;
  auto issue = [&](int k) {
    if (k - win_base >= 32) {
      win0 = win1;
      win_base += 32;
      win1 = win_base + 32 + lane < n_w ? stage_id(win_base + 32 + lane) : -1;
    }
    const int id = __shfl_sync(kFull, win0, k - win_base);  // k - win_base < 32 here
    if (lane == 0) {
      const int st = k % C::kStages;
      const int t0 = t_begin + (warp + kWarps * k) * kStageTokens;
      int row;
      if (id < 0 || id >= p.num_blocks) {
        flag_error(PKV_DEVERR_BLOCK_ID);
        row = p.num_blocks * p.bs;  // entirely out of bounds: TMA fills zeros
      } else {
        row = id * p.bs + t0 % p.bs;
      }
      mbar_arrive_expect_tx(&wbar[st], C::kStageBytes);
      C::load_stage(ring + st * C::kStageBytes, &tmK, &tmV, &wbar[st], kvh, row, pol);
    }
  };
  const int n_pro = n_w < C::kStages ? n_w : C::kStages;
  for (int k = 0; k < n_pro; ++k) issue(k);

  C c;
  if (it.prefix) c.init_gather(p, it.b0, it.members, kvh, lane);
  else c.init(p, it.b0, kvh, lane);
  for (int k = 0; k < n_w; ++k) {
    const int st = k % C::kStages;
    const bool ok = mbar_wait_bounded(&wbar[st], (uint32_t)((k / C::kStages) & 1));
    if (__any_sync(kFull, !ok)) {
      if (lane == 0) flag_error(PKV_DEVERR_TIMEOUT);
      for (int j = k; j < n_w && j < k + C::kStages; ++j)
        mbar_wait_bounded(&wbar[j % C::kStages], (uint32_t)((j / C::kStages) & 1));
      break;
    }
    const int t0 = t_begin + (warp + kWarps * k) * kStageTokens;
    c.consume(ring + st * C::kStageBytes, min(kStageTokens, t_end - t0), lane, [&] {
      if (k + C::kStages < n_w) issue(k + C::kStages);
    });
  }

  // Merge the warps; each row n = member * G + head goes to its sequence.
  c.store_state(reinterpret_cast<float*>(ring), lane);
  __syncthreads();
  constexpr int GP = C::GP;
  const int rows = it.members * G;
  const int SL = s.max_pp + s.max_op;
  for (int idx = threadIdx.x; idx < rows * D; idx += blockDim.x) {
    const int n = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, reinterpret_cast<const float*>(smem + w * kRing)[n]);
    float num = 0.f, den = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* stt = reinterpret_cast<const float*>(smem + w * kRing);
      const float f = exp2f(stt[n] - M);
      num = fmaf(f, stt[2 * GP + n * D + d], num);
      den = fmaf(f, stt[GP + n], den);
    }
    const int b = it.b0 + n / G, gg = n % G;
    if (pieces_of(s, b, it.plen, it.npp) == 1) {
      out[((size_t)b * p.Hq + (size_t)kvh * G + gg) * D + d] = __float2bfloat16_rn(num / den);
    } else {
      const size_t u = (((size_t)b * Hkv + kvh) * SL + it.slot) * G + gg;
      s.ws_acc[u * D + d] = num;
      if (d == 0) s.ws_ml[u] = make_float2(M, den);
    }
  }
  __threadfence();
  __syncthreads();

  // Tickets: the last piece of each (sequence, KV head) merges its partials.
  for (int i = 0; i < it.members; ++i) {
    const int b = it.b0 + i;
    const int tot = pieces_of(s, b, it.plen, it.npp);
    if (tot <= 1) continue;
    const size_t unit = (size_t)b * Hkv + kvh;
    if (threadIdx.x == 0) s_last = atomicAdd(&s.ws_count[unit], 1u) == (uint32_t)(tot - 1);
    __syncthreads();
    if (s_last) {
      __threadfence();
      const size_t base = unit * SL * G;
      auto slot_of = [&](int q) { return q < it.npp ? q : s.max_pp + (q - it.npp); };
      // As in the decode's merge: with at most 32 pieces, lane q reads piece q's
      // (max, sum) once and files its weight exp2(m_q - M) / den in the shared
      // memory the stages no longer use; then each thread sums 4-float chunks of
      // the output with kU pieces' loads in flight.
      constexpr int kU = 8;
      float* s_w = reinterpret_cast<float*>(smem);  // [piece][head]
      const bool fast = tot <= 32 && tot * G * (int)sizeof(float) <= DecodeSmem<C>::kRingBytes * kWarps &&
                        D % 4 == 0;
      for (int g = warp; g < G; g += kWarps) {
        float M = -INFINITY, den = 0.f;
        if (fast) {
          const float2 ml = lane < tot ? __ldcg(&s.ws_ml[base + (size_t)slot_of(lane) * G + g])
                                       : make_float2(-INFINITY, 0.f);
          M = ml.x;
#pragma unroll
          for (int off = 16; off >= 1; off /= 2) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
          const float e = lane < tot ? exp2f(ml.x - M) : 0.f;
          den = e * ml.y;
#pragma unroll
          for (int off = 16; off >= 1; off /= 2) den += __shfl_xor_sync(kFull, den, off);
          if (lane < tot) s_w[lane * G + g] = e / den;
        } else {
          for (int q = lane; q < tot; q += 32) M = fmaxf(M, __ldcg(&s.ws_ml[base + (size_t)slot_of(q) * G + g]).x);
#pragma unroll
          for (int off = 16; off >= 1; off /= 2) M = fmaxf(M, __shfl_xor_sync(kFull, M, off));
          for (int q = lane; q < tot; q += 32) {
            const float2 ml = __ldcg(&s.ws_ml[base + (size_t)slot_of(q) * G + g]);
            den += exp2f(ml.x - M) * ml.y;
          }
#pragma unroll
          for (int off = 16; off >= 1; off /= 2) den += __shfl_xor_sync(kFull, den, off);
        }
        if (lane == 0) {
          s_M[g] = M;
          s_den[g] = den;
        }
      }
      __syncthreads();
      T* o = out + ((size_t)b * p.Hq + (size_t)kvh * G) * D;
      if (fast) {
        for (int c = threadIdx.x; c < G * D / 4; c += blockDim.x) {
          const int g = c / (D / 4), d4 = c % (D / 4);
          float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int q0 = 0; q0 < tot; q0 += kU) {
            float4 v[kU];
#pragma unroll
            for (int k = 0; k < kU; ++k)
              v[k] = q0 + k < tot ? __ldcg(reinterpret_cast<const float4*>(
                                        s.ws_acc + (base + (size_t)slot_of(q0 + k) * G + g) * D) + d4)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < kU; ++k) {
              const float w = q0 + k < tot ? s_w[(q0 + k) * G + g] : 0.f;
              a.x = fmaf(w, v[k].x, a.x);
              a.y = fmaf(w, v[k].y, a.y);
              a.z = fmaf(w, v[k].z, a.z);
              a.w = fmaf(w, v[k].w, a.w);
            }
          }
          T* od = o + g * D + 4 * d4;
          od[0] = __float2bfloat16_rn(a.x);
          od[1] = __float2bfloat16_rn(a.y);
          od[2] = __float2bfloat16_rn(a.z);
          od[3] = __float2bfloat16_rn(a.w);
        }
      }
      for (int idx = threadIdx.x; !fast && idx < G * D; idx += blockDim.x) {
        const int g = idx / D, d = idx % D;
        float num = 0.f;
        for (int q = 0; q < tot; ++q) {
          const size_t u = base + (size_t)slot_of(q) * G + g;
          num = fmaf(exp2f(__ldcg(&s.ws_ml[u]).x - s_M[g]), __ldcg(&s.ws_acc[u * D + d]), num);
        }
        o[idx] = __float2bfloat16_rn(num / s_den[g]);
      }
      if (threadIdx.x == 0) s.ws_count[unit] = 0u;
    }
    __syncthreads();
  }
}

// Fused step of a group CTA (one KV head): every member's copy-on-write copy and
// new token row in one pass over all members.  Each element is written once: the
// copy leaves out the row that the new token fills, so no thread waits for another,
// and no member ever reads a row that another member is writing (in a fork the last
// holder writes its token into the block the others copy from, at the row they
// leave out).  The result equals copy_blocks then paged_kv_write.
// Member i's blocks come from the warp's per-member words in shared memory: its
// length (len), copy-on-write source (src, < 0: none) and row of the new token;
// dst[i] is the block the new token goes to (< 0: nothing to write), filed by
// resolve(), which runs once, after the first batch's reads are issued, so that
// those reads and the block ids share one memory latency.  The threads read up to
// kBatch elements each before writing any; the CTA's elements are taken in batches
// of kBatch x blockDim.x.
template <typename T, int D, class Resolve>
__device__ __forceinline__ void group_append(const DecodeParams& p, int lo, int members, int kvh,
                                             const int* len, const int* src, const int* row,
                                             const int* dst, Resolve&& resolve) {
  constexpr int kVec = D * (int)sizeof(T) / 16;  // 16-byte vectors per head row
  constexpr int kBatch = 8;
  const size_t row_vec = (size_t)p.Hkv * kVec;    // per token row (all heads)
  uint4* kc = reinterpret_cast<uint4*>(p.k_cache_w);
  uint4* vc = reinterpret_cast<uint4*>(p.v_cache_w);
  const uint4* kn = reinterpret_cast<const uint4*>(p.k_new);
  const uint4* vn = reinterpret_cast<const uint4*>(p.v_new);
  const int per = (p.bs + 1) * kVec;  // per member: the block's rows, then the new row
  const int total = members * per;
  bool resolved = false;
  for (int base = 0; base < total; base += kBatch * (int)blockDim.x) {
    uint4 ka[kBatch], va[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int x = base + j * (int)blockDim.x + (int)threadIdx.x;
      if (x >= total) break;
      const int i = x / per, r = (x % per) / kVec, c = x % kVec;
      if (len[i] <= 0) continue;
      if (r == p.bs) {
        const size_t so = ((size_t)(lo + i) * p.Hkv + kvh) * kVec + c;
        ka[j] = kn[so];
        va[j] = vn[so];
      } else if (src[i] >= 0 && r != row[i]) {
        const size_t so = ((size_t)src[i] * p.bs + r) * row_vec + (size_t)kvh * kVec + c;
        ka[j] = kc[so];
        va[j] = vc[so];
      }
    }
    if (!resolved) {
      resolve();
      resolved = true;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int x = base + j * (int)blockDim.x + (int)threadIdx.x;
      if (x >= total) break;
      const int i = x / per, r = (x % per) / kVec, c = x % kVec;
      const int d = dst[i];
      if (len[i] <= 0 || d < 0) continue;
      if (r == p.bs) {
        const size_t d_o = ((size_t)d * p.bs + row[i]) * row_vec + (size_t)kvh * kVec + c;
        kc[d_o] = ka[j];
        vc[d_o] = va[j];
      } else if (src[i] >= 0 && src[i] != d && r != row[i]) {
        const size_t d_o = ((size_t)d * p.bs + r) * row_vec + (size_t)kvh * kVec + c;
        kc[d_o] = ka[j];
        vc[d_o] = va[j];
      }
    }
  }
  if (!resolved) resolve();
  fence_proxy_async_global();
}

// A member's last stage when the fused step writes through the stages (blocks of
// 16 tokens, so the stage is the block): the new token's K and V rows go into row
// r of the stage in shared memory, in the 128-byte-swizzled layout the TMA boxes
// land in (16-byte chunk c of a row at position c ^ (row % 8) of its 64-dim
// sub-tile).  Then the block goes out to its destination d from there: all of it
// when it is a copy of block src (the stage was loaded from src), else row r
// alone.  Nothing in this launch reads those bytes of the pool again.  Each
// element of the pool is written once, as by copy_blocks then paged_kv_write.
template <class C, typename T, int D>
__device__ __forceinline__ void group_patch_stage(const DecodeParams& p, uint8_t* st,
                                                  const uint4* nrow, int r, int d, int src,
                                                  int kvh, int lane) {
  constexpr int kRowChunks = D * (int)sizeof(T) / 16;  // 16-byte chunks of one head row
  constexpr int kSub = kStageTokens * 128;             // one 64-dim sub-tile
  cp_async_wait_all();  // this lane's copies of the new rows; the barrier shows all
  __syncwarp();
  auto at = [&](int kv, int row, int cc) -> uint4* {
    return reinterpret_cast<uint4*>(st + kv * C::kTileBytes + (cc / 8) * kSub + row * 128 +
                                    (((cc % 8) ^ (row & 7)) << 4));
  };
  for (int x = lane; x < 2 * kRowChunks; x += 32) *at(x / kRowChunks, r, x % kRowChunks) = nrow[x];
  fence_proxy_async_smem();  // before the slot's next TMA fill
  __syncwarp();
  if (d < 0) return;
  uint4* kc = reinterpret_cast<uint4*>(p.k_cache_w);
  uint4* vc = reinterpret_cast<uint4*>(p.v_cache_w);
  const size_t row_vec = (size_t)p.Hkv * kRowChunks;  // per token row (all heads)
  const size_t head = (size_t)kvh * kRowChunks;
  if (src >= 0 && src != d) {
    for (int x = lane; x < 2 * kStageTokens * kRowChunks; x += 32) {
      const int kv = x / (kStageTokens * kRowChunks), rem = x % (kStageTokens * kRowChunks);
      const int row = rem / kRowChunks, cc = rem % kRowChunks;
      (kv ? vc : kc)[((size_t)d * kStageTokens + row) * row_vec + head + cc] = *at(kv, row, cc);
    }
  } else {
    for (int x = lane; x < 2 * kRowChunks; x += 32) {
      const int kv = x / kRowChunks, cc = x % kRowChunks;
      (kv ? vc : kc)[((size_t)d * kStageTokens + r) * row_vec + head + cc] = nrow[x];
    }
  }
}

// One CTA for a whole group and one KV head, when the group's members fit the
// 16 query rows of one MMA (members <= 16 / G).  The CTA's stages are the
// shared prefix's (scored for every member's rows) followed by each member's
// own tokens (scored for that member's rows only; the other rows see them as
// masked).  The warps take stages round-robin, so each warp's running softmax
// state covers some prefix stages and some own stages; merging the warps gives
// every row exactly its prefix plus its own tokens.  No partials leave the CTA.
// Shared memory of a group CTA: one slot per warp that holds its ring of
// stages and, at the end, its softmax state (M, l and O of 16 rows) for the
// merge; slots start on 1024-byte boundaries (the swizzled TMA boxes need it).
template <class C, int D, int W>
struct GroupSmem {
  static constexpr int kStateBytes = (2 * C::GP + C::GP * D) * 4;
  static constexpr int kRingBytes = DecodeSmem<C>::kRingBytes;
  static constexpr int kSlot =
      ((kRingBytes > kStateBytes ? kRingBytes : kStateBytes) + 1023) / 1024 * 1024;
  static constexpr size_t kBytes = 1024 /*alignment slack*/ + (size_t)W * kSlot + W * C::kStages * 8;
};

// The set-up takes two memory latencies before the stream runs: the first batch
// of loads (members' lengths, copy-on-write sources, the block ids of each warp's
// first prefix stages) is issued before any stage load, so that it does not queue
// behind them; each warp derives the prefix and the members' stage offsets from it
// on its own (no CTA barrier) and starts its first prefix stages.  The second batch
// (ids of own-token stages, the members' table check, the fused step's blocks and
// copy reads) runs while those stages are in flight.
// app_bar completes once every thread has made its share of the fused step's
// writes; only the loads of own-token stages wait for it.
template <class C, int D, int W>
__device__ __forceinline__ void group_piece(const SharedParams& s, int off_lo, int off_hi,
                                            int plen_req, int kvh, uint8_t* smem,
                                            uint64_t* app_bar, const CUtensorMap& tmK,
                                            const CUtensorMap& tmV) {
  using T = __nv_bfloat16;
  constexpr int kRing = GroupSmem<C, D, W>::kSlot;  // stride of the warps' slots
  constexpr int kMaxMembers = 16;
  static_assert(C::GP == 16, "group pieces use the 16-row consumer");
  // Each warp's own copy of the members' words: length, first stage (s_cum[i], with
  // s_cum[members] the CTA's stage count), copy-on-write source, new-token row and
  // block.
  __shared__ int s_len[W][kMaxMembers], s_cum[W][kMaxMembers + 1];
  __shared__ int s_src[W][kMaxMembers], s_row[W][kMaxMembers], s_dst[W][kMaxMembers];
  // Stage meta words (valid tokens | member << 5 | every-row flag << 10 | the
  // member's last stage << 11), filed by lane 0 beside the stage's slot when it
  // loads the stage.
  __shared__ int s_meta[W][C::kStages];
  // With 16-token blocks the fused step's writes go through the stages: the new
  // K and V rows of a member whose last stage a slot holds, copied in beside it.
  constexpr int kNewChunks = 2 * D * (int)sizeof(T) / 16;
  __shared__ uint4 s_new[W][C::kStages][kNewChunks];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + W * kRing);
  const DecodeParams& p = s.d;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int G = p.G;
  T* out = reinterpret_cast<T*>(p.out);
  // Group offsets are caller data: clamped into [0, B], so that no value of theirs
  // leads outside the batch.
  const int lo = min(max(off_lo, 0), p.B), hi = max(lo, min(max(off_hi, 0), p.B));
  int members = hi - lo;
  if (members <= 0) return;
  const int mc = min(s.mc, kMaxMembers);
  if (members > mc) {  // more members than the caller's bound: the rest stay unwritten
    if (threadIdx.x == 0) flag_error(PKV_DEVERR_PREFIX);
    members = mc;
  }
  uint8_t* ring = smem + warp * kRing;
  uint64_t* wbar = bars + warp * C::kStages;
  if (lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
#pragma unroll
    for (int st = 0; st < C::kStages; ++st) mbar_init(&wbar[st], 1);
    fence_mbar_init();
  }
  __syncwarp();
  const uint64_t pol = l2_policy_evict_first();
  const bool fused = p.k_new != nullptr;
  // A block is one stage: a member's last stage is loaded from its copy-on-write
  // source, the new row is put in place in shared memory, and the block is written
  // out from there (no copy pass, no wait on one).
  const bool patch = fused && p.bs == kStageTokens;
  const int32_t* r0 = p.block_tables + (size_t)lo * p.max_blocks;

  // First batch of loads.  Lane i: member i's length and copy-on-write source.  Every lane: the
  // block id of the warp's stage warp + W * lane, read as a prefix stage when the
  // caller's prefix reaches it (used only if the actual prefix does too).
  const int cap_pre = min(max(plen_req, 0), p.max_blocks * p.bs) / kStageTokens;
  const int kw = warp + W * lane;
  int win0p = kw < cap_pre ? r0[kw * kStageTokens / p.bs] : -1;
  int Li = 0, ci = -1;
  if (lane < members) {
    Li = shared_len(p, lo + lane);
    if (fused && p.cow_src != nullptr) ci = p.cow_src[lo + lane];
  }
  {  // the members' q rows of this KV head (read at the end of the set-up) into L2
    const int lines = G * D * (int)sizeof(T) / 128;  // per member, contiguous
    const uint8_t* q0 = reinterpret_cast<const uint8_t*>(p.q) +
                        ((size_t)lo * p.Hq + (size_t)kvh * G) * D * sizeof(T);
    for (int x = lane; x < members * lines; x += 32)
      prefetch_l2_line(q0 + (size_t)(x / lines) * p.Hq * D * sizeof(T) + (size_t)(x % lines) * 128);
  }
  // The prefix actually shared: short of every member's newest token (so no block
  // of it is one the fused step writes) and whole blocks.
  const int min_last = __reduce_min_sync(kFull, lane < members ? Li - 1 : 0x7fffffff);
  const int plen = max(0, min(plen_req, min_last)) / p.bs * p.bs;
  const int n_pre = plen / kStageTokens;
  int cum = (lane < members && Li > plen) ? (Li - plen + kStageTokens - 1) / kStageTokens : 0;
#pragma unroll
  for (int d = 1; d < 32; d *= 2) {
    const int y = __shfl_up_sync(kFull, cum, d);
    if (lane >= d) cum += y;
  }
  if (lane < members) {
    s_len[warp][lane] = Li;
    s_cum[warp][lane + 1] = n_pre + cum;
    s_src[warp][lane] = ci >= 0 && ci < p.num_blocks ? ci : -1;
    s_row[warp][lane] = Li > 0 ? (Li - 1) % p.bs : 0;
  }
  if (lane == 0) s_cum[warp][0] = n_pre;
  const int n_all = n_pre + __shfl_sync(kFull, cum, 31);
  __syncwarp();

  // This warp takes the CTA's stages warp, warp + W, ...; its stages win_base ..
  // win_base + 63 have their block ids resolved ahead, one per lane of two windows.
  // Window 0 holds prefix ids (win0p, first batch) and own-token ids (win0t, second batch)
  // apart, so that issuing a prefix stage never waits for a second-batch load.
  const int first = warp, stride = W;
  const int n_w = n_all > first ? (n_all - first + stride - 1) / stride : 0;
  auto stage_id = [&](int k) -> int {  // block id of the CTA's stage k, or -1
    if (k >= n_all) return -1;
    if (k < n_pre) return r0[k * kStageTokens / p.bs];
    int i = 0;
    while (k >= s_cum[warp][i + 1]) ++i;
    const int t0 = plen + (k - s_cum[warp][i]) * kStageTokens;
    return p.block_tables[(size_t)(lo + i) * p.max_blocks + t0 / p.bs];
  };
  int win_base = 0, win0t = -1, win1 = -1;
  bool app_seen = !fused || patch;  // lane 0: the fused step's writes are known to have landed
  auto issue = [&](int kk) {
    if (kk - win_base >= 32) {
      win0p = win1;
      win0t = win1;
      win_base += 32;
      win1 = stage_id(first + stride * (win_base + 32 + lane));
    }
    const int k = first + stride * kk;
    const int id = k < n_pre ? __shfl_sync(kFull, win0p, kk - win_base)
                             : __shfl_sync(kFull, win0t, kk - win_base);
    if (lane == 0) {
      if (k >= n_pre && !app_seen) {
        if (!mbar_wait_bounded(app_bar, 0)) flag_error(PKV_DEVERR_TIMEOUT);
        app_seen = true;
      }
      int t0, meta;
      if (k < n_pre) {
        t0 = k * kStageTokens;
        meta = kStageTokens | (1 << 10);  // every member's rows score it
      } else {
        int i = 0;
        while (k >= s_cum[warp][i + 1]) ++i;
        t0 = plen + (k - s_cum[warp][i]) * kStageTokens;
        meta = min(kStageTokens, s_len[warp][i] - t0) | (i << 5) | (members == 1 ? 1 << 10 : 0);
        if (patch && k == s_cum[warp][i + 1] - 1) meta |= 1 << 11;
      }
      int row = p.num_blocks * p.bs;  // past the pool: TMA fills zeros
      if (id < 0 || id >= p.num_blocks) {
        flag_error(PKV_DEVERR_BLOCK_ID);
      } else {
        row = id * p.bs + t0 % p.bs;
        const int src = (meta >> 11) ? s_src[warp][(meta >> 5) & 31] : -1;
        if (src >= 0 && src != id) row = src * p.bs;  // the block it is a copy of
      }
      const int st = kk % C::kStages;
      s_meta[warp][st] = meta;
      mbar_arrive_expect_tx(&wbar[st], C::kStageBytes);
      C::load_stage(ring + st * C::kStageBytes, &tmK, &tmV, &wbar[st], kvh, row, pol);
    }
    __syncwarp();  // the meta word is seen by every lane before the stage is consumed
    const int st = kk % C::kStages;
    const int m = s_meta[warp][st];
    if (m >> 11) {  // the member's new K and V rows, beside the slot
      const int i = (m >> 5) & 31;
      const uint4* kn = reinterpret_cast<const uint4*>(p.k_new);
      const uint4* vn = reinterpret_cast<const uint4*>(p.v_new);
      const size_t base = ((size_t)(lo + i) * p.Hkv + kvh) * (kNewChunks / 2);
      for (int x = lane; x < kNewChunks; x += 32)
        cp_async16(&s_new[warp][st][x],
                   x < kNewChunks / 2 ? kn + base + x : vn + base + x - kNewChunks / 2);
      cp_async_commit();
    }
  };
  // The first stages that lie in the prefix: a prefix block is never one that the
  // fused step writes.  They load after the second batch is issued, so that it does not
  // queue behind every warp's first stages.
  const int n_pro = n_w < C::kStages ? n_w : C::kStages;
  int n_early = 0;
  auto first_stages = [&] {
    while (n_early < n_pro && first + stride * n_early < n_pre) issue(n_early++);
  };

  // Second batch: ids of the own-token stages, the members' table check, and for a fused
  // step each member's new-token block and each thread's first copy reads.
  win0t = kw >= n_pre ? stage_id(kw) : -1;
  win1 = stage_id(first + stride * (32 + lane));
  // Every member must hold the same physical blocks for the prefix: entry j of
  // member i (i >= 1) against member 0's.  Two entries a thread are read now and
  // compared after the step's writes; the rest (long prefixes) after that.
  const int nj = plen / p.bs, n_chk = (members - 1) * nj;
  int chk_a[2] = {0, 0}, chk_b[2] = {0, 0};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int x = (int)threadIdx.x + j * (int)blockDim.x;
    if (x < n_chk) {
      chk_a[j] = p.block_tables[(size_t)(lo + 1 + x / nj) * p.max_blocks + x % nj];
      chk_b[j] = r0[x % nj];
    }
  }
  if (fused) {
    // Lane i: the block member i's new token goes to, filed before any write.
    int id = -1;
    if (lane < members && Li > 0)
      id = p.block_tables[(size_t)(lo + lane) * p.max_blocks + (Li - 1) / p.bs];
    auto resolve = [&] {
      first_stages();
      if (lane < members) {
        int d = -1;
        if (Li > 0) {
          if (id < 0 || id >= p.num_blocks) {
            if (warp == 0) flag_error(PKV_DEVERR_BLOCK_ID);
          } else {
            d = id;
            if (ci >= p.num_blocks && warp == 0) flag_error(PKV_DEVERR_COPY);
          }
        }
        s_dst[warp][lane] = d;
      }
      __syncwarp();
    };
    if (patch) {
      resolve();
    } else {
      group_append<T, D>(p, lo, members, kvh, s_len[warp], s_src[warp], s_row[warp],
                         s_dst[warp], resolve);
      mbar_arrive(app_bar);  // release: this thread's writes, fenced for the TMA reads
    }
  } else {
    first_stages();
  }
  bool chk_ok = chk_a[0] == chk_b[0] && chk_a[1] == chk_b[1];
  for (int x = (int)threadIdx.x + 2 * (int)blockDim.x; x < n_chk; x += blockDim.x)
    chk_ok &= p.block_tables[(size_t)(lo + 1 + x / nj) * p.max_blocks + x % nj] == r0[x % nj];
  if (!chk_ok) flag_error(PKV_DEVERR_PREFIX);
  while (n_early < n_pro) issue(n_early++);

  C c;
  c.init_gather(p, lo, members, kvh, lane);
  for (int kk = 0; kk < n_w; ++kk) {
    const int st = kk % C::kStages;
    const bool ok = mbar_wait_bounded(&wbar[st], (uint32_t)((kk / C::kStages) & 1));
    if (__any_sync(kFull, !ok)) {
      if (lane == 0) flag_error(PKV_DEVERR_TIMEOUT);
      for (int j = kk; j < n_w && j < kk + C::kStages; ++j)
        mbar_wait_bounded(&wbar[j % C::kStages], (uint32_t)((j / C::kStages) & 1));
      break;
    }
    const int meta = s_meta[warp][st];
    const int nv = meta & 31, r0 = ((meta >> 5) & 31) * G;
    if (meta >> 11)
      group_patch_stage<C, T, D>(p, ring + st * C::kStageBytes, s_new[warp][st], nv - 1,
                                 s_dst[warp][(meta >> 5) & 31], s_src[warp][(meta >> 5) & 31],
                                 kvh, lane);
    auto refill = [&] {
      if (kk + C::kStages < n_w) issue(kk + C::kStages);
    };
    if ((meta >> 10) & 1)  // every member's rows score it
      c.consume(ring + st * C::kStageBytes, nv, lane, refill);
    else
      c.consume_rows(ring + st * C::kStageBytes, nv, lane, r0, r0 + G, refill);
  }

  // Merge the warps; each row n = member * G + head goes to its sequence.  The
  // weights exp2(m_w - M) of each (warp, row) and 1 / l of each row are formed
  // once, then every thread combines 8 consecutive dims of one row.  A row with
  // no token at all (an empty sequence) is written as zeros.
  c.store_state(reinterpret_cast<float*>(ring), lane);
  __syncthreads();
  constexpr int GP = C::GP;
  __shared__ float s_wt[W][GP], s_inv[GP];
  auto state = [&](int w) { return reinterpret_cast<const float*>(smem + w * kRing); };
  const int rows = members * G;
  if (threadIdx.x < rows) {
    const int n = threadIdx.x;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < W; ++w) M = fmaxf(M, state(w)[n]);
    float den = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float f = M == -INFINITY ? 0.f : exp2f(state(w)[n] - M);
      s_wt[w][n] = f;
      den = fmaf(f, state(w)[GP + n], den);
    }
    s_inv[n] = den > 0.f ? 1.f / den : 0.f;
  }
  __syncthreads();
  constexpr int kChunks = D / 8;
  for (int idx = threadIdx.x; idx < rows * kChunks; idx += blockDim.x) {
    const int n = idx / kChunks, d0 = (idx % kChunks) * 8;
    float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < W; ++w) {
      const float f = s_wt[w][n];
      const float4* src = reinterpret_cast<const float4*>(state(w) + 2 * GP + n * D + d0);
      const float4 x = src[0], y = src[1];
      a[0] = fmaf(f, x.x, a[0]);
      a[1] = fmaf(f, x.y, a[1]);
      a[2] = fmaf(f, x.z, a[2]);
      a[3] = fmaf(f, x.w, a[3]);
      a[4] = fmaf(f, y.x, a[4]);
      a[5] = fmaf(f, y.y, a[5]);
      a[6] = fmaf(f, y.z, a[6]);
      a[7] = fmaf(f, y.w, a[7]);
    }
    const float inv = s_inv[n];
    uint4 v;
    v.x = pack_bf16x2(a[0] * inv, a[1] * inv);
    v.y = pack_bf16x2(a[2] * inv, a[3] * inv);
    v.z = pack_bf16x2(a[4] * inv, a[5] * inv);
    v.w = pack_bf16x2(a[6] * inv, a[7] * inv);
    *reinterpret_cast<uint4*>(out + ((size_t)(lo + n / G) * p.Hq + (size_t)kvh * G + n % G) * D +
                              d0) = v;
  }
}

// One CTA of W warps per (group, KV head): group_piece with consumer C (16 rows).
template <class C, int D, int W>
__global__ void __launch_bounds__(W * 32, D <= 128 ? 2 : 1)
    paged_decode_group_kernel(const SharedParams s, const __grid_constant__ CUtensorMap tmK,
                              const __grid_constant__ CUtensorMap tmV) {
  launch_overlap_entry();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int g = (int)blockIdx.x / s.d.Hkv, kvh = (int)blockIdx.x % s.d.Hkv;
  // The group's bounds and asked-for prefix are read before the timeout check, so
  // that the two latencies overlap.
  const int off_lo = s.group_offsets[g], off_hi = s.group_offsets[g + 1];
  const int plen_req = s.prefix_lens[g];
  __shared__ uint64_t s_app;  // the fused step's writes: one arrival per thread
  if (threadIdx.x == 0) {
    mbar_init(&s_app, W * 32);
    fence_mbar_init();
  }
  if (cta_timed_out()) return;  // its barrier also publishes the initialised s_app
  if (kvh == 0 && threadIdx.x == 0) {  // the groups must tile the batch in order
    bool ok = off_lo <= off_hi;
    if (g == 0) ok = ok && off_lo == 0;
    if (g == s.n_groups - 1) ok = ok && off_hi == s.d.B;
    if (!ok) flag_error(PKV_DEVERR_PREFIX);
  }
  group_piece<C, D, W>(s, off_lo, off_hi, plen_req, kvh, smem, &s_app, tmK, tmV);
}

template <class C2, class C1, int D>
__global__ void __launch_bounds__(kWarps * 32)
    paged_decode_shared_kernel(const SharedParams s, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV) {
  launch_overlap_entry();
  static_assert(DecodeSmem<C2>::kBytes == DecodeSmem<C1>::kBytes, "consumers share the ring");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  __shared__ float s_M[16], s_den[16];
  __shared__ int s_last;
  if (cta_timed_out()) return;
  if (blockIdx.x == 0 && threadIdx.x == 0) {  // the groups must tile the batch in order
    bool ok = s.group_offsets[0] == 0 && s.group_offsets[s.n_groups] == s.d.B;
    for (int g = 0; g < s.n_groups && ok; ++g) ok = s.group_offsets[g] <= s.group_offsets[g + 1];
    if (!ok) flag_error(PKV_DEVERR_PREFIX);
  }
  const SharedItem it = decode_shared_item(s, blockIdx.x);
  if (!it.valid) return;
  if (it.prefix) shared_piece<C2, D>(s, it, smem, tmK, tmV, s_M, s_den, s_last);
  else shared_piece<C1, D>(s, it, smem, tmK, tmV, s_M, s_den, s_last);
}

}  // namespace pkv
