// libpagedkv.so: C ABI (include/pagedkv.h) over the sm_100a kernels.
//
// Host side of every call: validate arguments (nothing is enqueued on an
// error), encode the TMA tensor maps for the decode, pick the kernel
// instantiation, launch on the caller's stream.
#include "pagedkv.h"

#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <mutex>
#include <utility>

#include "pkv_decode_balanced.cuh"
#include "pkv_decode_shared.cuh"
#include "pkv_prefill.cuh"
#include "pkv_write_copy.cuh"

namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<int> g_decode_path{PKV_PATH_AUTO};
std::atomic<int> g_decode_ctas{0};  // 0: as many as fit (at most 2 per SM)
std::atomic<int> g_decode_split{PKV_SPLIT_FIXED};
std::atomic<int> g_prefill_path{PKV_PREFILL_AUTO};

// SM count the partition choice is tuned for (B200).  It is a constant, not
// the device's attribute, so that the partition length and the workspace size
// stay pure functions of the arguments (no CUDA call, no device state): the
// caller can size a workspace before choosing a device or stream.  On a
// device with another SM count the choice stays correct, only its wave count
// is tuned for 148 SMs.
constexpr int kSmCount = 148;

// Multiprocessors of the current device (looked up once per device).
cudaError_t sm_count(int* out) {
  static std::atomic<int> cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 0 && dev < 64 && cache[dev].load() > 0) {
    *out = cache[dev].load();
    return cudaSuccess;
  }
  e = cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev);
  if (e == cudaSuccess && dev >= 0 && dev < 64) cache[dev].store(*out);
  return e;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int cuda_fail(cudaError_t e) {
  g_last_cuda_error = static_cast<int>(e);
  return PKV_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Tensor maps.  The pool [num_blocks][bs][Hkv][D] is viewed as a 3-D tensor
// {D, Hkv, num_blocks*bs} (innermost first); one box is 16 token rows of one
// KV head: {D or 64, 1, 16}.  Its x coordinate is always 0 or a multiple of 64
// elements, so every box starts on a 16-byte boundary.
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int make_cache_map(CUtensorMap* map, const void* base, int D, int Hkv, int64_t rows,
                   pkv_dtype dtype, bool swizzle, int box_rows = pkv::kStageTokens) {
  auto fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  const int es = dtype == PKV_BF16 ? 2 : 4;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)Hkv * D * es};
  cuuint32_t box[3] = {(cuuint32_t)(swizzle ? 64 : D), 1u, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(map, dtype == PKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                         : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {  // reported as 100000 + the driver's CUresult
    g_last_cuda_error = 100000 + static_cast<int>(r);
    return PKV_ERR_CUDA;
  }
  return PKV_OK;
}

// Map of a bf16 cache for the tensor-core decode kernels: 4-D (64 dims,
// tokens, 64-dim halves, KV heads) with a box of {64, 16, D / 64, 1}, so that
// one TMA load brings a 16-token tile as D / 64 swizzled 16 x 128 B sub-tiles.
// The dims of one token are contiguous, so its halves lie 128 bytes apart.
// `half_box` (8-token blocks): a box of {64, 8, 1, 1}, one half of one sub-tile.
int make_stage_map(CUtensorMap* map, const void* base, int D, int Hkv, int64_t rows,
                   pkv_dtype dtype, bool half_box = false) {
  if (dtype != PKV_BF16 || D % 64 != 0) return PKV_ERR_UNSUPPORTED;
  auto fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[4] = {64u, (cuuint64_t)rows, (cuuint64_t)(D / 64), (cuuint64_t)Hkv};
  cuuint64_t strides[3] = {(cuuint64_t)Hkv * D * 2, 128u, (cuuint64_t)D * 2};
  cuuint32_t box[4] = {64u, (cuuint32_t)(half_box ? pkv::kStageTokens / 2 : pkv::kStageTokens),
                       (cuuint32_t)(half_box ? 1 : D / 64), 1u};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {  // reported as 100000 + the driver's CUresult
    g_last_cuda_error = 100000 + static_cast<int>(r);
    return PKV_ERR_CUDA;
  }
  return PKV_OK;
}

// Launches a kernel with programmatic stream serialization: its CTAs may be placed
// while the kernel before it in the stream finishes (once that kernel's CTAs have
// all begun), and each waits in launch_overlap_entry() for that kernel to complete
// before it touches global memory.  Back-to-back steps thus overlap one grid's
// launch and CTA set-up with the previous grid's last CTAs.  Returns the launch's
// error, else any earlier asynchronous one.
std::atomic<int> g_launch_overlap{1};  // pkv_set_launch_overlap

template <typename... Params, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = g_launch_overlap.load(std::memory_order_relaxed) ? 1 : 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  return e != cudaSuccess ? e : cudaGetLastError();
}

// Raises the dynamic shared-memory limit of a kernel once per device.  `done`
// must be distinct for every kernel (all decode kernels share one C++ type).
template <typename Kernel>
int ensure_smem(Kernel kernel, size_t bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return PKV_OK;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return cuda_fail(e);
  done.fetch_or(bit, std::memory_order_acq_rel);
  return PKV_OK;
}

int auto_partition(int B, int Hkv, int max_seq_len) {
  // About half the longest sequence, between 512 and 4096 tokens: the longest
  // sequences are cut in two (halving the largest CTAs, which set the tail)
  // while most sequences stay whole.  Longer partitions waste less on
  // start-up and on partial results; every partition costs a CTA start-up
  // (table ids, q, pipeline fill) and a partial write and merge.  Then shorten
  // until there are about three waves of CTAs (3 resident per SM).  Measured on
  // B200: MHA (max 2049) best at 1024, GQA (max 4097) at 2048, long context
  // (max 131073) at 4096.
  const int64_t units = (int64_t)B * Hkv;
  const int64_t target = (int64_t)kSmCount * 3 * 3;
  const int64_t L = max_seq_len > 0 ? max_seq_len : 1;
  int P = 512;  // the power of two nearest (in log scale) to L / 2
  while (P < 4096 && (double)L / 2 >= (double)P * 1.4142135623730951) P *= 2;
  while (P > 512 && units * ceil_div(L, P) < target) P /= 2;
  return P;
}

struct DecodeShape {
  bool balanced;  // work-balanced persistent kernel (else fixed-length partitions)
  int P;          // partition length of the fixed split (0 when balanced)
  int max_parts;
  size_t off_ml, off_acc, bytes;  // workspace layout and size of the split in use
  size_t ws_bytes;                // size reported to callers: covers either split
};

// `fused` (paged_decode_step): fixed-length partitions whatever the split mode,
// and a partition length rounded up to whole blocks.  The step rewrites the
// block that receives each sequence's new token (copy-on-write copy and the new
// row) from the CTA of the sequence's last partition, so no other partition may
// hold tokens of that block.  `fixed_only`: fixed-length partitions, nothing else.
int decode_shape(int B, int Hq, int Hkv, int D, int max_seq_len, int block_size,
                 int partition_size, DecodeShape* s, bool fused = false,
                 bool fixed_only = false) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || max_seq_len < 0)
    return PKV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return PKV_ERR_INVALID_ARG;
  if (partition_size < 0 || partition_size % pkv::kStageTokens != 0) return PKV_ERR_INVALID_ARG;
  const size_t G = (size_t)(Hq / Hkv);
  const size_t units = (size_t)B * Hkv;
  auto align256 = [](size_t x) { return (x + 255) & ~(size_t)255; };

  // Fixed-length partitions (the default split).
  int P = partition_size > 0 ? partition_size : auto_partition(B, Hkv, max_seq_len);
  if (fused && P % block_size != 0) P = (int)ceil_div(P, block_size) * block_size;
  const int64_t mp = max_seq_len > 0 ? ceil_div(max_seq_len, P) : 1;
  if (mp > 65535) return PKV_ERR_OUT_OF_RANGE;
  size_t f_ml = 0, f_acc = 0, f_bytes = 0;
  if (mp > 1 && B > 0) {
    f_ml = align256(units * sizeof(uint32_t));
    f_acc = f_ml + align256(units * mp * G * sizeof(float2));
    f_bytes = f_acc + units * mp * G * (size_t)D * sizeof(float);
  }
  // Work-balanced split (opt-in): needs the per-sequence prefix in shared memory
  // and a stage count that fits in 31 bits.
  const int64_t max_stages = (int64_t)B * Hkv * ceil_div(max_seq_len, pkv::kStageTokens);
  const bool bal_ok = partition_size == 0 && B <= pkv::kBalancedMaxB && max_stages < 0x7fffffffLL &&
                      block_size % pkv::kStageTokens == 0;
  size_t b_ml = 0, b_acc = 0, b_bytes = 0;
  if (bal_ok && B > 0) {
    const size_t slots = pkv::balanced_slots((size_t)B, (size_t)Hkv);
    b_ml = align256(units * sizeof(uint32_t));
    b_acc = b_ml + align256(slots * G * sizeof(float2));
    b_bytes = b_acc + slots * G * (size_t)D * sizeof(float);
  }
  s->balanced = bal_ok && !fused && !fixed_only &&
                g_decode_split.load(std::memory_order_relaxed) == PKV_SPLIT_BALANCED;
  s->P = s->balanced ? 0 : P;
  s->max_parts = s->balanced ? 0 : (int)mp;
  s->off_ml = s->balanced ? b_ml : f_ml;
  s->off_acc = s->balanced ? b_acc : f_acc;
  s->bytes = s->balanced ? b_bytes : f_bytes;
  s->ws_bytes = std::max(f_bytes, b_bytes);
  return PKV_OK;
}

template <class C, typename T, int D, int LAYOUT>
int launch_decode(const pkv::DecodeParams& p, int B, const CUtensorMap& mk, const CUtensorMap& mv,
                  cudaStream_t stream) {
  auto kernel = pkv::paged_decode_kernel<C, T, D, LAYOUT>;
  const size_t smem = pkv::DecodeSmem<C>::kBytes;
  static std::atomic<uint64_t> smem_set{0};
  int rc = ensure_smem(kernel, smem, smem_set);
  if (rc != PKV_OK) return rc;
  dim3 grid((unsigned)p.Hkv, (unsigned)p.max_parts, (unsigned)B);
  cudaError_t e = launch_overlapped(kernel, grid, dim3(pkv::kWarps * 32), smem, stream, p, mk, mv);
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

// Balanced kernel: a persistent grid of as many CTAs as are resident at once
// (at most 2 per SM), so that every worker starts at the same time.
template <class C, typename T, int D>
int launch_balanced(const pkv::DecodeParams& p, const CUtensorMap& mk, const CUtensorMap& mv,
                    cudaStream_t stream) {
  auto kernel = pkv::paged_decode_balanced_kernel<C, T, D>;
  static std::atomic<uint64_t> smem_set{0};
  static std::atomic<int> resident[64];
  int rc = ensure_smem(kernel, pkv::BalancedSmem<C>::bytes(pkv::kBalancedMaxB), smem_set);
  if (rc != PKV_OK) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  int ctas = resident[dev & 63].load(std::memory_order_relaxed);
  if (ctas == 0) {
    int sms = 0, per_sm = 0;
    e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
        &per_sm, kernel, pkv::kWarps * 32, pkv::BalancedSmem<C>::bytes(pkv::kBalancedMaxB));
    if (e != cudaSuccess) return cuda_fail(e);
    ctas = std::max(1, std::min(sms * std::min(per_sm, 2), pkv::kBalancedMaxCtas));
    resident[dev & 63].store(ctas, std::memory_order_relaxed);
  }
  const int forced = g_decode_ctas.load(std::memory_order_relaxed);
  if (forced > 0) ctas = std::min(forced, pkv::kBalancedMaxCtas);
  e = launch_overlapped(kernel, dim3(ctas), dim3(pkv::kWarps * 32), pkv::BalancedSmem<C>::bytes(p.B),
                        stream, p, mk, mv);
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

// The balanced split exists for the plain block layout only (decode_shape never
// picks it for another layout).
template <class C, typename T, int D, int LAYOUT>
int launch_any(const pkv::DecodeParams& p, bool balanced, const CUtensorMap& mk,
               const CUtensorMap& mv, cudaStream_t s) {
  if constexpr (LAYOUT == pkv::kLayoutPaged) {
    if (balanced) return launch_balanced<C, T, D>(p, mk, mv, s);
  }
  return launch_decode<C, T, D, LAYOUT>(p, p.B, mk, mv, s);
}

template <typename T, int D, int LAYOUT>
int dispatch_simt(const pkv::DecodeParams& p, bool bal, const CUtensorMap& mk,
                  const CUtensorMap& mv, cudaStream_t s) {
  if (p.G == 1) return launch_any<pkv::SimtConsumer<T, D, 1>, T, D, LAYOUT>(p, bal, mk, mv, s);
  if (p.G == 2) return launch_any<pkv::SimtConsumer<T, D, 2>, T, D, LAYOUT>(p, bal, mk, mv, s);
  if (p.G <= 4) return launch_any<pkv::SimtConsumer<T, D, 4>, T, D, LAYOUT>(p, bal, mk, mv, s);
  if (p.G <= 8) return launch_any<pkv::SimtConsumer<T, D, 8>, T, D, LAYOUT>(p, bal, mk, mv, s);
  return PKV_ERR_UNSUPPORTED;
}

template <int D, int LAYOUT>
int dispatch_mma(const pkv::DecodeParams& p, bool bal, const CUtensorMap& mk,
                 const CUtensorMap& mv, cudaStream_t s) {
  using T = __nv_bfloat16;
  if (p.G <= 8) return launch_any<pkv::MmaConsumer<D, 1>, T, D, LAYOUT>(p, bal, mk, mv, s);
  if (p.G <= 16) return launch_any<pkv::MmaConsumer<D, 2>, T, D, LAYOUT>(p, bal, mk, mv, s);
  return PKV_ERR_UNSUPPORTED;
}

// bf16 runs on the tensor-core consumer by default, whatever G: its work per
// 16-token stage does not depend on G (heads are padded to 8), and it issues
// far fewer, shorter dependency chains than the CUDA-core consumer (measured on
// B200, MHA workload: 6.71 vs 4.53 TB/s).
bool use_tensor_cores(pkv_dtype dtype, int G) {
  if (dtype != PKV_BF16) return false;
  const int mode = g_decode_path.load(std::memory_order_relaxed);
  if (mode == PKV_PATH_CUDA_CORES) return G > 8;  // CUDA-core kernels stop at G = 8
  return true;
}

// Shared-prefix decode: partition length, slots and workspace layout.
struct SharedShape {
  int P, max_pp, max_op, SL;
  size_t off_ml, off_acc, bytes;
};

// `fused` (paged_decode_step_shared_prefix): the partition length is rounded up to
// whole blocks, so that the block receiving a sequence's new token lies in its
// last own partition only (see decode_shape).
int shared_shape(int B, int Hq, int Hkv, int D, int max_seq_len, int block_size,
                 int partition_size, SharedShape* s, bool fused = false) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || max_seq_len < 0)
    return PKV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return PKV_ERR_INVALID_ARG;
  if (partition_size < 0 || partition_size % pkv::kStageTokens != 0) return PKV_ERR_INVALID_ARG;
  // Prefix pieces carry most of the bytes, and each is read once for up to 16
  // query rows; long partitions keep their count (and the partials) low.
  // Measured on B200 (shared-prefix workloads): 2048 beats 1024 and 512.
  s->P = partition_size > 0 ? partition_size : std::max(2048, auto_partition(B, Hkv, max_seq_len));
  if (fused && s->P % block_size != 0) s->P = (int)ceil_div(s->P, block_size) * block_size;
  const int64_t mp = std::max<int64_t>(1, ceil_div(max_seq_len, s->P));
  if (mp > 32767) return PKV_ERR_OUT_OF_RANGE;
  s->max_pp = (int)mp;
  s->max_op = (int)mp;
  s->SL = 2 * (int)mp;
  const size_t G = (size_t)(Hq / Hkv);
  const size_t units = (size_t)B * Hkv;
  auto align256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  s->off_ml = align256(units * sizeof(uint32_t));
  s->off_acc = s->off_ml + align256(units * s->SL * G * sizeof(float2));
  s->bytes = B == 0 ? 0 : s->off_acc + units * s->SL * G * (size_t)D * sizeof(float);
  return PKV_OK;
}

// Prefix pieces stack up to 16 query rows (two 8-row MMA tiles); own pieces
// need only G rows, so they run the one-tile consumer when G <= 8.
template <int D, int NT_OWN>
int launch_shared(const pkv::SharedParams& sp, int64_t items, const CUtensorMap& mk,
                  const CUtensorMap& mv, cudaStream_t stream) {
  using C2 = pkv::MmaConsumer<D, 2>;
  using C1 = pkv::MmaConsumer<D, NT_OWN>;
  auto kernel = pkv::paged_decode_shared_kernel<C2, C1, D>;
  const size_t smem = pkv::DecodeSmem<C2>::kBytes;
  static std::atomic<uint64_t> smem_set{0};
  int rc = ensure_smem(kernel, smem, smem_set);
  if (rc != PKV_OK) return rc;
  cudaError_t e = launch_overlapped(kernel, dim3((unsigned)items), dim3(pkv::kWarps * 32), smem,
                                    stream, sp, mk, mv);
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

// One CTA of GROUP_WARPS warps per (group, KV head), 16-row consumer with a
// ring of GROUP_STAGES stages per warp (D = 128; other head dims: 6 warps and
// the consumer's default ring).  Measured on B200 (share workloads): 6 warps
// (2 CTAs per SM) beat 4 by up to 7% and 8 (1 CTA per SM) are 1.3x slower;
// 3 stages equal 2, 4 stages (1 CTA per SM) are 1.6x slower.  At 160 registers
// a thread two CTAs of 6 warps fill an SM's register file.
#ifndef PKV_GROUP_STAGES_D128
#define PKV_GROUP_STAGES_D128 2
#endif
#ifndef PKV_GROUP_WARPS_D128
#define PKV_GROUP_WARPS_D128 6
#endif
template <int D>
int launch_group(const pkv::SharedParams& sp, int64_t items, const CUtensorMap& mk,
                 const CUtensorMap& mv, cudaStream_t stream) {
  constexpr int kStages = D == 128 ? PKV_GROUP_STAGES_D128 : pkv::MmaConsumer<D, 2>::kStages;
  constexpr int W = D == 128 ? PKV_GROUP_WARPS_D128 : 6;
  using C = pkv::MmaConsumer<D, 2, kStages>;
  auto kernel = pkv::paged_decode_group_kernel<C, D, W>;
  const size_t smem = pkv::GroupSmem<C, D, W>::kBytes;
  static std::atomic<uint64_t> smem_set{0};
  int rc = ensure_smem(kernel, smem, smem_set);
  if (rc != PKV_OK) return rc;
  cudaError_t e = launch_overlapped(kernel, dim3((unsigned)items), dim3(W * 32), smem, stream, sp,
                                    mk, mv);
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

int paged_kv_write(const void* k, const void* v, void* k_cache, void* v_cache,
                   const int64_t* slot_mapping, int64_t N, int Hkv, int D, int block_size,
                   int64_t num_blocks, pkv_dtype dtype, pkv_stream_t stream) {
  if (dtype != PKV_BF16 && dtype != PKV_F32) return PKV_ERR_INVALID_ARG;
  if (N < 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || num_blocks <= 0) return PKV_ERR_INVALID_ARG;
  if (N == 0) return PKV_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
    return PKV_ERR_INVALID_ARG;
  const int64_t es = dtype == PKV_BF16 ? 2 : 4;
  const int64_t row_bytes = (int64_t)Hkv * D * es;
  if (row_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
  if (N > 0x7fffffffLL) return PKV_ERR_OUT_OF_RANGE;
  if (num_blocks > (INT64_MAX / block_size) / row_bytes) return PKV_ERR_OUT_OF_RANGE;
  const int64_t row_vec = row_bytes / 16;
  const int threads = 256;
  const int64_t gy = std::min<int64_t>(std::max<int64_t>(ceil_div(row_vec, threads), 1), 65535);
  dim3 grid((unsigned)N, (unsigned)gy);
  cudaError_t e = launch_overlapped(
      pkv::kv_write_kernel, grid, dim3(threads), 0, stream, static_cast<const uint4*>(k),
      static_cast<const uint4*>(v), static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
      slot_mapping, row_vec, num_blocks * block_size);
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

int paged_attention_decode_partition_size(int B, int Hkv, int max_seq_len, int block_size,
                                          int partition_size) {
  DecodeShape s;
  const int rc = decode_shape(B, Hkv, Hkv, 16, max_seq_len, block_size, partition_size, &s);
  return rc == PKV_OK ? s.P : rc;
}

size_t paged_attention_decode_workspace_size(int B, int Hq, int Hkv, int D, int max_seq_len,
                                             int block_size, int partition_size) {
  DecodeShape s;
  if (decode_shape(B, Hq, Hkv, D, max_seq_len, block_size, partition_size, &s) != PKV_OK) return 0;
  return s.ws_bytes;
}

}  // extern "C"

namespace {

// The fused step's extra inputs (all null for a plain decode), and the flag of
// the unpaged control (paged_attention_decode_contiguous).
struct StepArgs {
  const void* k_new = nullptr;
  const void* v_new = nullptr;
  const int32_t* cow_src = nullptr;
  bool contiguous = false;
};

template <int LAYOUT>
int dispatch_layout(const pkv::DecodeParams& p, bool tc, bool bal, pkv_dtype dtype, int D,
                    const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t stream) {
  if (tc) {
    if (D == 64) return dispatch_mma<64, LAYOUT>(p, bal, mk, mv, stream);
    if (D == 128) return dispatch_mma<128, LAYOUT>(p, bal, mk, mv, stream);
    return dispatch_mma<256, LAYOUT>(p, bal, mk, mv, stream);
  }
  if constexpr (LAYOUT == pkv::kLayoutContig) {
    return PKV_ERR_UNSUPPORTED;  // the unpaged control runs the tensor-core kernels only
  } else {
    if (dtype == PKV_BF16) {
      if (D == 64) return dispatch_simt<__nv_bfloat16, 64, LAYOUT>(p, bal, mk, mv, stream);
      if (D == 128) return dispatch_simt<__nv_bfloat16, 128, LAYOUT>(p, bal, mk, mv, stream);
      return dispatch_simt<__nv_bfloat16, 256, LAYOUT>(p, bal, mk, mv, stream);
    }
    if (D == 64) return dispatch_simt<float, 64, LAYOUT>(p, bal, mk, mv, stream);
    return dispatch_simt<float, 128, LAYOUT>(p, bal, mk, mv, stream);
  }
}

int decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                int max_seq_len, int B, int Hq, int Hkv, int D, int block_size,
                int64_t num_blocks, float scale, pkv_dtype dtype, int partition_size,
                void* workspace, size_t workspace_bytes, pkv_stream_t stream,
                const StepArgs& step) {
  const bool fused = step.k_new != nullptr;
  const bool contig = step.contiguous;
  if (dtype != PKV_BF16 && dtype != PKV_F32) return PKV_ERR_INVALID_ARG;
  DecodeShape shape;
  int rc = decode_shape(B, Hq, Hkv, D, max_seq_len, block_size, partition_size, &shape, fused,
                        contig);
  if (rc != PKV_OK) return rc;
  if (max_blocks <= 0 || num_blocks <= 0 || !std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
  if (B == 0) return PKV_OK;
  if (B > 65535) return PKV_ERR_OUT_OF_RANGE;
  if (!out || !q || !k_cache || !v_cache || (!block_tables && !contig) || !seq_lens)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return PKV_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  const bool d_ok = dtype == PKV_BF16 ? (D == 64 || D == 128 || D == 256) : (D == 64 || D == 128);
  if (!d_ok) return PKV_ERR_UNSUPPORTED;
  // Blocks of 8 tokens (a 16-token stage from two blocks) or multiples of 16.
  const bool bs8 = !contig && block_size == pkv::kStageTokens / 2;
  if (!contig && !bs8 && (block_size % pkv::kStageTokens != 0 || block_size > 256))
    return PKV_ERR_UNSUPPORTED;
  if (G > (dtype == PKV_BF16 ? 16 : 8)) return PKV_ERR_UNSUPPORTED;
  if (num_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_seq_len > (int64_t)max_blocks * block_size) return PKV_ERR_OUT_OF_RANGE;
  if (shape.bytes > 0) {
    if (!workspace || workspace_bytes < shape.bytes) return PKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PKV_ERR_WORKSPACE;
  }

  if (fused && (!step.v_new || !aligned16(step.k_new) || !aligned16(step.v_new) ||
                (reinterpret_cast<uintptr_t>(step.cow_src) & 3u)))
    return PKV_ERR_INVALID_ARG;
  pkv::DecodeParams p{};
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ws_count = shape.bytes ? reinterpret_cast<uint32_t*>(ws) : nullptr;
  p.ws_ml = shape.bytes ? reinterpret_cast<float2*>(ws + shape.off_ml) : nullptr;
  p.ws_acc = shape.bytes ? reinterpret_cast<float*>(ws + shape.off_acc) : nullptr;
  p.B = B;
  p.max_blocks = max_blocks;
  p.max_seq_len = max_seq_len;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.bs = block_size;
  p.part_tokens = shape.P;
  p.max_parts = shape.max_parts;
  p.num_blocks = (int)num_blocks;
  p.scale_log2 = scale * 1.4426950408889634f;
  // A few sequences cut into long partitions: CTAs in length order, so that the
  // shortest start last (measured on the long-context workload).
  p.sorted = !shape.balanced && B <= pkv::kSortedMaxB && shape.P >= 2048 ? 1 : 0;
  if (fused) {
    p.k_new = step.k_new;
    p.v_new = step.v_new;
    p.k_cache_w = const_cast<void*>(k_cache);
    p.v_cache_w = const_cast<void*>(v_cache);
    p.cow_src = step.cow_src;
  }

  const bool tc = use_tensor_cores(dtype, G);
  if (contig && !tc) return PKV_ERR_UNSUPPORTED;
  CUtensorMap mk, mv;
  const int64_t rows = num_blocks * block_size;
  const int box_rows = bs8 ? pkv::kStageTokens / 2 : pkv::kStageTokens;
  if ((rc = tc ? make_stage_map(&mk, k_cache, D, Hkv, rows, dtype, bs8)
                : make_cache_map(&mk, k_cache, D, Hkv, rows, dtype, false, box_rows)) != PKV_OK)
    return rc;
  if ((rc = tc ? make_stage_map(&mv, v_cache, D, Hkv, rows, dtype, bs8)
                : make_cache_map(&mv, v_cache, D, Hkv, rows, dtype, false, box_rows)) != PKV_OK)
    return rc;

  const bool bal = shape.balanced;
  if (contig) return dispatch_layout<pkv::kLayoutContig>(p, tc, false, dtype, D, mk, mv, stream);
  if (bs8) return dispatch_layout<pkv::kLayoutPaged8>(p, tc, false, dtype, D, mk, mv, stream);
  return dispatch_layout<pkv::kLayoutPaged>(p, tc, bal, dtype, D, mk, mv, stream);
}

}  // namespace

extern "C" {

int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                           int max_seq_len, int B, int Hq, int Hkv, int D, int block_size,
                           int64_t num_blocks, float scale, pkv_dtype dtype, int partition_size,
                           void* workspace, size_t workspace_bytes, pkv_stream_t stream) {
  return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks, seq_lens, max_seq_len, B,
                     Hq, Hkv, D, block_size, num_blocks, scale, dtype, partition_size, workspace,
                     workspace_bytes, stream, StepArgs{});
}

int paged_attention_decode_contiguous(void* out, const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* seq_lens,
                                      int max_seq_len, int row_stride, int B, int Hq, int Hkv,
                                      int D, float scale, pkv_dtype dtype, int partition_size,
                                      void* workspace, size_t workspace_bytes,
                                      pkv_stream_t stream) {
  if (row_stride <= 0 || row_stride < max_seq_len) return PKV_ERR_INVALID_ARG;
  if (dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  StepArgs contig;
  contig.contiguous = true;
  // Sequence b is "block" b of row_stride tokens, and the kernel never reads a table.
  return decode_impl(out, q, k_cache, v_cache, nullptr, 1, seq_lens, max_seq_len, B, Hq, Hkv, D,
                     row_stride, std::max(B, 1), scale, dtype, partition_size, workspace,
                     workspace_bytes, stream, contig);
}

int paged_decode_step(void* out, const void* q, const void* k_new, const void* v_new,
                      void* k_cache, void* v_cache, const int32_t* block_tables, int max_blocks,
                      const int32_t* seq_lens, const int32_t* cow_src, int max_seq_len, int B,
                      int Hq, int Hkv, int D, int block_size, int64_t num_blocks, float scale,
                      pkv_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
                      pkv_stream_t stream) {
  if (!k_new || !v_new) return PKV_ERR_INVALID_ARG;
  StepArgs step;
  step.k_new = k_new;
  step.v_new = v_new;
  step.cow_src = cow_src;
  return decode_impl(out, q, k_cache, v_cache, block_tables, max_blocks, seq_lens, max_seq_len, B,
                     Hq, Hkv, D, block_size, num_blocks, scale, dtype, partition_size, workspace,
                     workspace_bytes, stream, step);
}

size_t paged_attention_decode_shared_prefix_workspace_size(int B, int Hq, int Hkv, int D,
                                                           int max_seq_len, int block_size,
                                                           int partition_size) {
  SharedShape s;
  if (shared_shape(B, Hq, Hkv, D, max_seq_len, block_size, partition_size, &s) != PKV_OK) return 0;
  return s.bytes;
}

}  // extern "C"

namespace {

int shared_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                int max_seq_len, const int32_t* group_offsets, const int32_t* prefix_lens,
                int n_groups, int max_group_size, int B, int Hq, int Hkv, int D, int block_size,
                int64_t num_blocks, float scale, pkv_dtype dtype, int partition_size,
                void* workspace, size_t workspace_bytes, pkv_stream_t stream,
                const StepArgs& step) {
  if (dtype != PKV_BF16 && dtype != PKV_F32) return PKV_ERR_INVALID_ARG;
  SharedShape shape;
  int rc = shared_shape(B, Hq, Hkv, D, max_seq_len, block_size, partition_size, &shape,
                        step.k_new != nullptr);
  if (rc != PKV_OK) return rc;
  if (max_blocks <= 0 || num_blocks <= 0 || !std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
  if (n_groups <= 0 || max_group_size <= 0) return PKV_ERR_INVALID_ARG;
  if (B == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !group_offsets ||
      !prefix_lens)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) ||
      (reinterpret_cast<uintptr_t>(group_offsets) & 3u) ||
      (reinterpret_cast<uintptr_t>(prefix_lens) & 3u))
    return PKV_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (D != 64 && D != 128 && D != 256) return PKV_ERR_UNSUPPORTED;
  if (block_size % pkv::kStageTokens != 0 || block_size > 256) return PKV_ERR_UNSUPPORTED;
  if (G > 16) return PKV_ERR_UNSUPPORTED;
  if (num_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_seq_len > (int64_t)max_blocks * block_size) return PKV_ERR_OUT_OF_RANGE;
  if (max_group_size > B) max_group_size = B;
  if (shape.bytes > 0) {
    if (!workspace || workspace_bytes < shape.bytes) return PKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PKV_ERR_WORKSPACE;
  }
  const int mc = std::max(1, 16 / G);
  const int64_t chunks = ceil_div(max_group_size, mc);
  const int64_t prefix_items = (int64_t)n_groups * chunks * shape.max_pp * Hkv;
  // A group whose members fit one MMA chunk is one CTA per KV head (prefix and
  // own tokens together, no partials) unless the caller fixed a partition length.
  const bool grouped = partition_size == 0 && max_group_size <= mc;
  const int64_t items = grouped ? (int64_t)n_groups * Hkv
                                : prefix_items + (int64_t)n_groups * max_group_size * shape.max_op * Hkv;
  if (items > 0x7fffffffLL) return PKV_ERR_OUT_OF_RANGE;

  if (step.k_new && (!step.v_new || !aligned16(step.k_new) || !aligned16(step.v_new) ||
                     (reinterpret_cast<uintptr_t>(step.cow_src) & 3u)))
    return PKV_ERR_INVALID_ARG;
  pkv::SharedParams sp{};
  pkv::DecodeParams& p = sp.d;
  p.k_new = step.k_new;
  p.v_new = step.v_new;
  p.k_cache_w = step.k_new ? const_cast<void*>(k_cache) : nullptr;
  p.v_cache_w = step.k_new ? const_cast<void*>(v_cache) : nullptr;
  p.cow_src = step.cow_src;
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.ws_acc = nullptr;
  p.ws_ml = nullptr;
  p.ws_count = nullptr;
  p.B = B;
  p.max_blocks = max_blocks;
  p.max_seq_len = max_seq_len;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.bs = block_size;
  p.part_tokens = shape.P;
  p.max_parts = shape.max_op;
  p.num_blocks = (int)num_blocks;
  p.scale_log2 = scale * 1.4426950408889634f;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  sp.group_offsets = group_offsets;
  sp.prefix_lens = prefix_lens;
  sp.ws_count = reinterpret_cast<uint32_t*>(ws);
  sp.ws_ml = reinterpret_cast<float2*>(ws + shape.off_ml);
  sp.ws_acc = reinterpret_cast<float*>(ws + shape.off_acc);
  sp.n_groups = n_groups;
  sp.chunks = (int)chunks;
  sp.mc = mc;
  sp.max_pp = shape.max_pp;
  sp.max_op = shape.max_op;
  sp.max_group = max_group_size;
  sp.P = shape.P;
  sp.n_prefix_items = (int)prefix_items;

  CUtensorMap mk, mv;
  const int64_t rows = num_blocks * block_size;
  if ((rc = make_stage_map(&mk, k_cache, D, Hkv, rows, dtype)) != PKV_OK) return rc;
  if ((rc = make_stage_map(&mv, v_cache, D, Hkv, rows, dtype)) != PKV_OK) return rc;
  if (grouped) {
    if (D == 64) return launch_group<64>(sp, items, mk, mv, stream);
    if (D == 128) return launch_group<128>(sp, items, mk, mv, stream);
    return launch_group<256>(sp, items, mk, mv, stream);
  }
  if (G <= 8) {
    if (D == 64) return launch_shared<64, 1>(sp, items, mk, mv, stream);
    if (D == 128) return launch_shared<128, 1>(sp, items, mk, mv, stream);
    return launch_shared<256, 1>(sp, items, mk, mv, stream);
  }
  if (D == 64) return launch_shared<64, 2>(sp, items, mk, mv, stream);
  if (D == 128) return launch_shared<128, 2>(sp, items, mk, mv, stream);
  return launch_shared<256, 2>(sp, items, mk, mv, stream);
}

}  // namespace

extern "C" {

int paged_attention_decode_shared_prefix(void* out, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* block_tables,
                                         int max_blocks, const int32_t* seq_lens, int max_seq_len,
                                         const int32_t* group_offsets, const int32_t* prefix_lens,
                                         int n_groups, int max_group_size, int B, int Hq, int Hkv,
                                         int D, int block_size, int64_t num_blocks, float scale,
                                         pkv_dtype dtype, int partition_size, void* workspace,
                                         size_t workspace_bytes, pkv_stream_t stream) {
  return shared_impl(out, q, k_cache, v_cache, block_tables, max_blocks, seq_lens, max_seq_len,
                     group_offsets, prefix_lens, n_groups, max_group_size, B, Hq, Hkv, D,
                     block_size, num_blocks, scale, dtype, partition_size, workspace,
                     workspace_bytes, stream, StepArgs{});
}

int paged_decode_step_shared_prefix(void* out, const void* q, const void* k_new, const void* v_new,
                                    void* k_cache, void* v_cache, const int32_t* block_tables,
                                    int max_blocks, const int32_t* seq_lens, const int32_t* cow_src,
                                    int max_seq_len, const int32_t* group_offsets,
                                    const int32_t* prefix_lens, int n_groups, int max_group_size,
                                    int B, int Hq, int Hkv, int D, int block_size,
                                    int64_t num_blocks, float scale, pkv_dtype dtype,
                                    int partition_size, void* workspace, size_t workspace_bytes,
                                    pkv_stream_t stream) {
  if (!k_new || !v_new) return PKV_ERR_INVALID_ARG;
  StepArgs step;
  step.k_new = k_new;
  step.v_new = v_new;
  step.cow_src = cow_src;
  return shared_impl(out, q, k_cache, v_cache, block_tables, max_blocks, seq_lens, max_seq_len,
                     group_offsets, prefix_lens, n_groups, max_group_size, B, Hq, Hkv, D,
                     block_size, num_blocks, scale, dtype, partition_size, workspace,
                     workspace_bytes, stream, step);
}

size_t paged_attention_prefill_workspace_size(int B, int Hq, int Hkv, int max_q_len) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || max_q_len <= 0 || Hq % Hkv != 0) return 0;
  const int G = Hq / Hkv;
  if (G > pkv::kPrefillRows) return 0;
  const int64_t nqt = ceil_div(max_q_len, 2 * (pkv::kPrefillRows / G));
  const int64_t items = (int64_t)B * nqt * Hkv;
  if (items > 0x7fffffffLL) return 0;
  return (size_t)(2 + items) * sizeof(int32_t);
}

int paged_attention_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                            const int32_t* cu_q, int total_q, int max_q_len, int max_seq_len,
                            int B, int Hq, int Hkv, int D, int block_size, int64_t num_blocks,
                            float scale, pkv_dtype dtype, void* workspace,
                            size_t workspace_bytes, pkv_stream_t stream) {
  if (dtype != PKV_BF16 && dtype != PKV_F32) return PKV_ERR_INVALID_ARG;
  if (B < 0 || total_q < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0 ||
      max_blocks <= 0 || num_blocks <= 0 || max_seq_len < 0 || max_q_len < 0 ||
      !std::isfinite(scale) || Hq % Hkv != 0)
    return PKV_ERR_INVALID_ARG;
  if (B == 0 || total_q == 0) return PKV_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !cu_q)
    return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(cu_q) & 3u))
    return PKV_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  if (dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
  if (D != 64 && D != 128 && D != 256) return PKV_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return PKV_ERR_UNSUPPORTED;
  if (block_size % pkv::kStageTokens != 0 || block_size > 256) return PKV_ERR_UNSUPPORTED;
  if (max_q_len < 1 || max_q_len > max_seq_len) return PKV_ERR_OUT_OF_RANGE;
  if (num_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_seq_len > (int64_t)max_blocks * block_size) return PKV_ERR_OUT_OF_RANGE;
  const int TQ = pkv::kPrefillRows / G;
  // Two query tiles per CTA on the warp-specialised kernel (D <= 128, which
  // leaves TMEM room for both tiles' S and O); one on the single-tile kernel.
  const bool two_tile = D <= 128 && g_prefill_path != PKV_PREFILL_SINGLE_TILE;
  const int64_t q_tiles = ceil_div(max_q_len, two_tile ? 2 * TQ : TQ);
  if (B > 65535 || q_tiles > 65535) return PKV_ERR_OUT_OF_RANGE;
  if (workspace) {
    if ((reinterpret_cast<uintptr_t>(workspace) & 3u) ||
        workspace_bytes < paged_attention_prefill_workspace_size(B, Hq, Hkv, max_q_len))
      return PKV_ERR_INVALID_ARG;
  }

  pkv::PrefillParams p{};
  p.out = out;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  p.cu_q = cu_q;
  p.max_blocks = max_blocks;
  p.max_seq_len = max_seq_len;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = G;
  p.TQ = TQ;
  p.bs = block_size;
  p.num_blocks = (int)num_blocks;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.nqt = (int)q_tiles;
  p.n_items = (int)((int64_t)B * q_tiles * Hkv);
  p.sched = nullptr;

  // Query rows [T][Hq][D] as a 3-D tensor {D, Hq, T}; one box = 128 rows of one
  // KV head: {64, G, 128 / G}, 128-byte swizzled (the K-major MMA operand).
  auto fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  CUtensorMap mq, mk, mv;
  cuuint64_t qdims[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)total_q};
  cuuint64_t qstrides[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
  cuuint32_t qbox[3] = {64u, (cuuint32_t)G, (cuuint32_t)TQ};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), qdims, qstrides,
                  qbox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = 100000 + static_cast<int>(r);
    return PKV_ERR_CUDA;
  }
  int rc;
  const int64_t rows = num_blocks * block_size;
  if ((rc = make_cache_map(&mk, k_cache, D, Hkv, rows, dtype, true)) != PKV_OK) return rc;
  if ((rc = make_cache_map(&mv, v_cache, D, Hkv, rows, dtype, true)) != PKV_OK) return rc;
  dim3 grid((unsigned)Hkv, (unsigned)q_tiles, (unsigned)B);
  auto launch = [&](auto kernel, size_t smem, std::atomic<uint64_t>& set, int threads) -> int {
    int rc2 = ensure_smem(kernel, smem, set);
    if (rc2 != PKV_OK) return rc2;
    cudaError_t e = launch_overlapped(kernel, grid, dim3(threads), smem, stream, p, mq, mk, mv);
    return e == cudaSuccess ? PKV_OK : cuda_fail(e);
  };
  static std::atomic<uint64_t> pp64{0}, pp128{0}, set64{0}, set128{0}, set256{0};
  if (two_tile) {
    // With a workspace: order the items longest first, then one persistent CTA
    // per SM takes them in that order.  Without: one CTA per item.
    if (workspace) {
      p.sched = static_cast<int*>(workspace);
      cudaError_t e = launch_overlapped(pkv::prefill_schedule_kernel, dim3(1),
                                        dim3(pkv::kSchedThreads), 0, stream, p);
      if (e != cudaSuccess) return cuda_fail(e);
      int sms = 0;
      if ((e = sm_count(&sms)) != cudaSuccess) return cuda_fail(e);
      grid = dim3((unsigned)std::min<int64_t>(sms, p.n_items), 1, 1);
    }
    if (D == 64)
      return launch(pkv::paged_prefill_pp_kernel<64>, pkv::PpSmem<64>::kBytes, pp64, pkv::kPpThreads);
    return launch(pkv::paged_prefill_pp_kernel<128>, pkv::PpSmem<128>::kBytes, pp128, pkv::kPpThreads);
  }
  const int th = pkv::kWarps * 32;
  if (D == 64) return launch(pkv::paged_prefill_kernel<64>, pkv::PrefillSmem<64>::kBytes, set64, th);
  if (D == 128)
    return launch(pkv::paged_prefill_kernel<128>, pkv::PrefillSmem<128>::kBytes, set128, th);
  return launch(pkv::paged_prefill_kernel<256>, pkv::PrefillSmem<256>::kBytes, set256, th);
}

int copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping, int64_t P,
                int64_t block_bytes, int64_t num_blocks, pkv_stream_t stream) {
  if (P < 0 || block_bytes <= 0 || num_blocks <= 0) return PKV_ERR_INVALID_ARG;
  if (P == 0) return PKV_OK;
  if (!k_cache || !v_cache || !block_mapping) return PKV_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(block_mapping) & 7u))
    return PKV_ERR_INVALID_ARG;
  if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
  if (P > 0x7fffffffLL) return PKV_ERR_OUT_OF_RANGE;
  if (num_blocks > INT64_MAX / block_bytes) return PKV_ERR_OUT_OF_RANGE;
  const int64_t block_vec = block_bytes / 16;
  const int threads = 256;
  const int64_t gy = std::min<int64_t>(std::max<int64_t>(ceil_div(block_vec, threads * 4), 1), 65535);
  dim3 grid((unsigned)P, (unsigned)gy);
  cudaError_t e = launch_overlapped(pkv::copy_blocks_kernel, grid, dim3(threads), 0, stream,
                                    static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache),
                                    block_mapping, block_vec, num_blocks);
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

// ---------------------------------------------------------------------------
// Allocation-free decode.  Its scratch is this file-scope device array.  In
// host code the symbol is only a stand-in for the array; the device address
// comes from cudaGetSymbolAddress, looked up once per device.
// ---------------------------------------------------------------------------
}  // extern "C"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

int noalloc_scratch(void** ptr) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return PKV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return PKV_OK;
}

}  // namespace

extern "C" {

int paged_attention_decode_noalloc(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   int max_blocks, const int32_t* seq_lens, int max_seq_len, int B,
                                   int Hq, int Hkv, int D, int block_size, int64_t num_blocks,
                                   float scale, pkv_dtype dtype, int partition_size,
                                   pkv_stream_t stream) {
  DecodeShape shape;
  int rc = decode_shape(B, Hq, Hkv, D, max_seq_len, block_size, partition_size, &shape);
  if (rc != PKV_OK) return rc;
  if (shape.bytes > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  if (shape.bytes > 0) {
    if ((rc = noalloc_scratch(&scratch)) != PKV_OK) return rc;
    // The partition counters must start at zero; the array keeps whatever the
    // previous call left, so clear them on this call's stream first.
    cudaError_t e = cudaMemsetAsync(scratch, 0, shape.off_ml, stream);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return paged_attention_decode(out, q, k_cache, v_cache, block_tables, max_blocks, seq_lens,
                                max_seq_len, B, Hq, Hkv, D, block_size, num_blocks, scale, dtype,
                                partition_size, scratch, shape.bytes > 0 ? PKV_NOALLOC_SCRATCH_BYTES : 0,
                                stream);
}

const char* pkv_status_string(int status) {
  switch (status) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_OUT_OF_RANGE: return "size or bound out of range";
    case PKV_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case PKV_ERR_CUDA: return "CUDA error (see pkv_last_cuda_error)";
    case PKV_ERR_UNSUPPORTED: return "unsupported shape";
    case PKV_ERR_SCRATCH_LIMIT: return "sizes need more scratch than the allocation-free decode has";
    default: return "unknown status";
  }
}

int pkv_last_cuda_error(void) { return g_last_cuda_error; }

int pkv_device_errors(uint32_t* bits, int clear) {
  if (!bits) return PKV_ERR_INVALID_ARG;
  cudaError_t e = cudaMemcpyFromSymbol(bits, pkv::g_device_errors, sizeof(uint32_t));
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    const uint32_t zero = 0;
    e = cudaMemcpyToSymbol(pkv::g_device_errors, &zero, sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return PKV_OK;
}

int pkv_set_decode_split(int mode) {
  if (mode != PKV_SPLIT_FIXED && mode != PKV_SPLIT_BALANCED) return PKV_ERR_INVALID_ARG;
  return g_decode_split.exchange(mode);
}

int pkv_set_decode_ctas(int ctas) {
  if (ctas < 0) return PKV_ERR_INVALID_ARG;
  return g_decode_ctas.exchange(ctas);
}

namespace pkv {
// One thread waits, with the bounded wait of every pipeline, on a barrier that
// nothing completes; it gives up after the time limit and flags the timeout.
__global__ void stalled_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait_bounded(&bar, 0)) flag_error(PKV_DEVERR_TIMEOUT);
  }
}
}  // namespace pkv

int pkv_debug_stalled_wait(pkv_stream_t stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  pkv::stalled_wait_kernel<<<1, 32, 0, stream>>>();
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

int pkv_set_prefill_path(int mode) {
  if (mode != PKV_PREFILL_AUTO && mode != PKV_PREFILL_SINGLE_TILE) return PKV_ERR_INVALID_ARG;
  return g_prefill_path.exchange(mode);
}

int pkv_set_launch_overlap(int enabled) {
  if (enabled != 0 && enabled != 1) return PKV_ERR_INVALID_ARG;
  return g_launch_overlap.exchange(enabled);
}

int pkv_set_decode_path(int mode) {
  if (mode != PKV_PATH_AUTO && mode != PKV_PATH_CUDA_CORES && mode != PKV_PATH_TENSOR_CORES)
    return PKV_ERR_INVALID_ARG;
  return g_decode_path.exchange(mode);
}

}  // extern "C"
