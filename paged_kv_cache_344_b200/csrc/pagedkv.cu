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

#include "pkv_write_copy.cuh"

namespace {

thread_local int g_last_cuda_error = 0;
std::atomic<int> g_decode_path{PKV_PATH_AUTO};

constexpr int kSmCount = 148;  // B200

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
                   pkv_dtype dtype, bool swizzle) {
  auto fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  const int es = dtype == PKV_BF16 ? 2 : 4;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)Hkv, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * es, (cuuint64_t)Hkv * D * es};
  cuuint32_t box[3] = {(cuuint32_t)(swizzle ? 64 : D), 1u, (cuuint32_t)pkv::kStageTokens};
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
  // Long partitions: every CTA pays a start-up (table ids, q, pipeline fill)
  // and every extra partition a partial write and merge, and CTAs whose
  // partition lies past a short sequence's end still occupy a slot briefly.
  // Shorten them only until there are about three waves of CTAs
  // (2 resident per SM).  Measured on B200: 4096 beats 2048, 1024 and 512 on
  // the MHA, GQA and long-context workloads.
  const int64_t units = (int64_t)B * Hkv;
  const int64_t target = (int64_t)kSmCount * 2 * 3;
  int P = 4096;
  while (P > 512 && units * ceil_div(max_seq_len > 0 ? max_seq_len : 1, P) < target) P /= 2;
  return P;
}

struct DecodeShape {
  int P;
  int max_parts;
  size_t off_ml, off_acc, bytes;
};

int decode_shape(int B, int Hq, int Hkv, int D, int max_seq_len, int block_size,
                 int partition_size, DecodeShape* s) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0 || max_seq_len < 0)
    return PKV_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return PKV_ERR_INVALID_ARG;
  if (partition_size < 0 || partition_size % pkv::kStageTokens != 0) return PKV_ERR_INVALID_ARG;
  const int P = partition_size > 0 ? partition_size : auto_partition(B, Hkv, max_seq_len);
  const int64_t mp = max_seq_len > 0 ? ceil_div(max_seq_len, P) : 1;
  if (mp > 65535) return PKV_ERR_OUT_OF_RANGE;
  s->P = P;
  s->max_parts = (int)mp;
  if (mp <= 1 || B == 0) {
    s->off_ml = s->off_acc = s->bytes = 0;
    return PKV_OK;
  }
  const size_t G = (size_t)(Hq / Hkv);
  const size_t units = (size_t)B * Hkv;
  auto align256 = [](size_t x) { return (x + 255) & ~(size_t)255; };
  s->off_ml = align256(units * sizeof(uint32_t));
  s->off_acc = s->off_ml + align256(units * mp * G * sizeof(float2));
  s->bytes = s->off_acc + units * mp * G * (size_t)D * sizeof(float);
  return PKV_OK;
}

template <class C, typename T, int D>
int launch_decode(const pkv::DecodeParams& p, int B, const CUtensorMap& mk, const CUtensorMap& mv,
                  cudaStream_t stream) {
  auto kernel = pkv::paged_decode_kernel<C, T, D>;
  const size_t smem = pkv::DecodeSmem<C>::kBytes;
  static std::atomic<uint64_t> smem_set{0};
  int rc = ensure_smem(kernel, smem, smem_set);
  if (rc != PKV_OK) return rc;
  dim3 grid((unsigned)p.Hkv, (unsigned)p.max_parts, (unsigned)B);
  kernel<<<grid, pkv::kWarps * 32, smem, stream>>>(p, mk, mv);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? PKV_OK : cuda_fail(e);
}

template <typename T, int D>
int dispatch_simt(const pkv::DecodeParams& p, int B, const CUtensorMap& mk,
                  const CUtensorMap& mv, cudaStream_t s) {
  if (p.G == 1) return launch_decode<pkv::SimtConsumer<T, D, 1>, T, D>(p, B, mk, mv, s);
  if (p.G == 2) return launch_decode<pkv::SimtConsumer<T, D, 2>, T, D>(p, B, mk, mv, s);
  if (p.G <= 4) return launch_decode<pkv::SimtConsumer<T, D, 4>, T, D>(p, B, mk, mv, s);
  if (p.G <= 8) return launch_decode<pkv::SimtConsumer<T, D, 8>, T, D>(p, B, mk, mv, s);
  return PKV_ERR_UNSUPPORTED;
}

template <int D>
int dispatch_mma(const pkv::DecodeParams& p, int B, const CUtensorMap& mk, const CUtensorMap& mv,
                 cudaStream_t s) {
  if (p.G <= 8)
    return launch_decode<pkv::MmaConsumer<D, 1>, __nv_bfloat16, D>(p, B, mk, mv, s);
  if (p.G <= 16)
    return launch_decode<pkv::MmaConsumer<D, 2>, __nv_bfloat16, D>(p, B, mk, mv, s);
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
  pkv::kv_write_kernel<<<grid, threads, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, row_vec, num_blocks * block_size);
  cudaError_t e = cudaGetLastError();
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
  return s.bytes;
}

int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                           int max_seq_len, int B, int Hq, int Hkv, int D, int block_size,
                           int64_t num_blocks, float scale, pkv_dtype dtype, int partition_size,
                           void* workspace, size_t workspace_bytes, pkv_stream_t stream) {
  if (dtype != PKV_BF16 && dtype != PKV_F32) return PKV_ERR_INVALID_ARG;
  DecodeShape shape;
  int rc = decode_shape(B, Hq, Hkv, D, max_seq_len, block_size, partition_size, &shape);
  if (rc != PKV_OK) return rc;
  if (max_blocks <= 0 || num_blocks <= 0 || !std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
  if (B == 0) return PKV_OK;
  if (B > 65535) return PKV_ERR_OUT_OF_RANGE;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PKV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) ||
      (reinterpret_cast<uintptr_t>(block_tables) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
    return PKV_ERR_INVALID_ARG;
  const int G = Hq / Hkv;
  const bool d_ok = dtype == PKV_BF16 ? (D == 64 || D == 128 || D == 256) : (D == 64 || D == 128);
  if (!d_ok) return PKV_ERR_UNSUPPORTED;
  if (block_size % pkv::kStageTokens != 0 || block_size > 256) return PKV_ERR_UNSUPPORTED;
  if (G > (dtype == PKV_BF16 ? 16 : 8)) return PKV_ERR_UNSUPPORTED;
  if (num_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_blocks > 0x7fffffffLL / block_size) return PKV_ERR_OUT_OF_RANGE;
  if ((int64_t)max_seq_len > (int64_t)max_blocks * block_size) return PKV_ERR_OUT_OF_RANGE;
  if (shape.bytes > 0) {
    if (!workspace || workspace_bytes < shape.bytes) return PKV_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) & 255u) return PKV_ERR_WORKSPACE;
  }

  pkv::DecodeParams p;
  p.out = out;
  p.q = q;
  p.block_tables = block_tables;
  p.seq_lens = seq_lens;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ws_count = shape.bytes ? reinterpret_cast<uint32_t*>(ws) : nullptr;
  p.ws_ml = shape.bytes ? reinterpret_cast<float2*>(ws + shape.off_ml) : nullptr;
  p.ws_acc = shape.bytes ? reinterpret_cast<float*>(ws + shape.off_acc) : nullptr;
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

  const bool tc = use_tensor_cores(dtype, G);
  CUtensorMap mk, mv;
  const int64_t rows = num_blocks * block_size;
  if ((rc = make_cache_map(&mk, k_cache, D, Hkv, rows, dtype, tc)) != PKV_OK) return rc;
  if ((rc = make_cache_map(&mv, v_cache, D, Hkv, rows, dtype, tc)) != PKV_OK) return rc;

  if (tc) {
    if (D == 64) return dispatch_mma<64>(p, B, mk, mv, stream);
    if (D == 128) return dispatch_mma<128>(p, B, mk, mv, stream);
    return dispatch_mma<256>(p, B, mk, mv, stream);
  }
  if (dtype == PKV_BF16) {
    if (D == 64) return dispatch_simt<__nv_bfloat16, 64>(p, B, mk, mv, stream);
    if (D == 128) return dispatch_simt<__nv_bfloat16, 128>(p, B, mk, mv, stream);
    return dispatch_simt<__nv_bfloat16, 256>(p, B, mk, mv, stream);
  }
  if (D == 64) return dispatch_simt<float, 64>(p, B, mk, mv, stream);
  return dispatch_simt<float, 128>(p, B, mk, mv, stream);
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
  pkv::copy_blocks_kernel<<<grid, threads, 0, stream>>>(static_cast<uint4*>(k_cache),
                                                        static_cast<uint4*>(v_cache),
                                                        block_mapping, block_vec, num_blocks);
  cudaError_t e = cudaGetLastError();
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

int pkv_set_decode_path(int mode) {
  if (mode != PKV_PATH_AUTO && mode != PKV_PATH_CUDA_CORES && mode != PKV_PATH_TENSOR_CORES)
    return PKV_ERR_INVALID_ARG;
  return g_decode_path.exchange(mode);
}

}  // extern "C"
