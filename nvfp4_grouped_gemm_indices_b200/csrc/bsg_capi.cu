// bsg_capi.cu -- the extern "C" boundary of libbsg.so: argument checks, TMA descriptor encoding,
// tactic choice and kernel launch.  Declarations and the full contract are in include/bsg.h.
//
// The argument checks follow the host binding of the page "[flashinfer] FlashInfer FP8 GEMM 최적화:
// 윈도우 세그먼트 KG1 프로그램으로 GPU 성능 극대화", section 1 (rank and unit-inner-stride checks,
// K % 128, 16-byte strides and base addresses, boxes larger than an extent only on axes that may run
// past the end, descriptive messages) and the launch contract of its section 2 (1 <= M <= 2^24,
// 64 <= N <= 2^19).  Nothing is launched when a check fails.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>

#include "../../include/bsg.h"
#include "bsg_quant.cuh"
#include "bsg_chooser.h"
#include "bsg_fp8.cuh"
#include "bsg_fp8_swap.cuh"
#include "bsg_moe.cuh"
#include "bsg_nvfp4.cuh"

#define BSG_VERSION_STRING "bsg 0.1.0 (sm_100a)"

namespace {

thread_local std::string g_last_error;

bsg_status fail(bsg_status code, const char* fmt, ...) {
  char buf[1024];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

__device__ bsg::DeviceStatus g_device_status;

uint64_t g_timeout_ns = 2000000000ull;
int g_debug_fault = 0;
std::mutex g_mu;

constexpr int kMaxDevices = 64;
struct DeviceState {
  bool ready = false;
  int sm_count = 0;
  bsg::DeviceStatus* status = nullptr;
  bool fp8_attr = false;
  bool fp8_swap_attr = false;
  bool fp8_n64_attr = false;
  bool nvfp4_attr = false;
  bool moe_attr = false;
  int fp8_pair_clusters = 0;
  int nvfp4_pair_clusters = 0;
};
DeviceState g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bsg_status cuda_fail(cudaError_t e, const char* what) {
  return fail(BSG_ERR_CUDA, "%s failed: %s (%d)", what, cudaGetErrorString(e), static_cast<int>(e));
}

// Per-device set-up (once per device, with that device current): SM count, the device address of
// the status word, the kernels' shared-memory attribute.
bsg_status device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BSG_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    int major = 0, minor = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(major)");
    if ((e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(minor)");
    if (major != 10 || minor != 0)
      return fail(BSG_ERR_CUDA, "device %d is sm_%d%d; this library is built for sm_100a (B200) only", dev, major,
                  minor);
    if ((e = cudaDeviceGetAttribute(&st.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    void* addr = nullptr;
    if ((e = cudaGetSymbolAddress(&addr, g_device_status)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress(status word)");
    st.status = static_cast<bsg::DeviceStatus*>(addr);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return fail(BSG_ERR_CUDA, "cannot resolve cuTensorMapEncodeTiled from the driver");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    st.ready = true;
  }
  *out = &st;
  return BSG_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Encodes a tiled descriptor after the same checks as the page's binding: extents >= box unless the
// axis may run past the end, strides multiples of 16 bytes, 16-byte aligned base.
struct DescKey {
  const void* base;
  int rank;
  int swz;
  uint64_t dims[5];
  uint64_t strides[4];
  uint32_t box[5];
};
struct DescCacheEntry {
  DescKey key;
  CUtensorMap map;
  bool valid = false;
};
constexpr int kDescCacheSize = 8;

bsg_status encode(CUtensorMap* map, const char* name, const void* base, int rank, const uint64_t* dims,
                  const uint64_t* strides_bytes, const uint32_t* box, const bool* allow_oob,
                  CUtensorMapSwizzle swz) {
  if (!aligned(base, 16)) return fail(BSG_ERR_ALIGNMENT, "operand %s: base address must be 16-byte aligned", name);
  for (int i = 0; i < rank; ++i) {
    if (dims[i] == 0 || dims[i] > (1ull << 32))
      return fail(BSG_ERR_UNSUPPORTED_SHAPE, "operand %s: extent %llu on axis %d outside [1, 2^32]", name,
                  static_cast<unsigned long long>(dims[i]), i);
    if (!allow_oob[i] && box[i] > dims[i])
      return fail(BSG_ERR_UNSUPPORTED_SHAPE,
                  "operand %s: axis %d (0 = innermost) has a TMA box of %u elements but the extent is %llu; "
                  "this axis may not run past its end",
                  name, i, box[i], static_cast<unsigned long long>(dims[i]));
  }
  for (int i = 0; i + 1 < rank; ++i) {
    if (strides_bytes[i] % 16 != 0 || strides_bytes[i] >= (1ull << 40))
      return fail(BSG_ERR_ALIGNMENT, "operand %s: stride %llu bytes (axis %d) must be a multiple of 16 below 2^40",
                  name, static_cast<unsigned long long>(strides_bytes[i]), i + 1);
  }
  // A descriptor depends only on these arguments: repeated calls on the same buffers (the common case
  // in a serving loop) reuse the last encodings of the calling thread instead of re-encoding.
  DescKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = rank;
  key.swz = static_cast<int>(swz);
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) key.strides[i] = strides_bytes[i];
  thread_local DescCacheEntry cache[kDescCacheSize];
  thread_local int next_victim = 0;
  for (int i = 0; i < kDescCacheSize; ++i) {
    if (cache[i].valid && memcmp(&cache[i].key, &key, sizeof(key)) == 0) {
      *map = cache[i].map;
      return BSG_OK;
    }
  }
  cuuint64_t gdim[5], gstr[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    gdim[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) gstr[i] = strides_bytes[i];
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                        gdim, gstr, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(BSG_ERR_CUDA, "cuTensorMapEncodeTiled of %s failed (CUresult %d)", name, (int)r);
  DescCacheEntry& e = cache[next_victim];
  next_victim = (next_victim + 1) % kDescCacheSize;
  e.key = key;
  e.map = *map;
  e.valid = true;
  return BSG_OK;
}

bsg_status check_common(const void* A, const void* B, const int32_t* m_indices, const void* C, int64_t M, int64_t N,
                        int64_t K, int64_t G) {
  if (!A || !B || !C) return fail(BSG_ERR_INVALID_ARG, "A, B and C must be non-null device pointers");
  if (G < 1 || G > 4096) return fail(BSG_ERR_UNSUPPORTED_SHAPE, "G = %lld outside [1, 4096]", (long long)G);
  if (!m_indices && G != 1)
    return fail(BSG_ERR_INVALID_ARG, "m_indices may be NULL only when G == 1 (G = %lld)", (long long)G);
  if (M < 1 || M > (1ll << 24))
    return fail(BSG_ERR_UNSUPPORTED_SHAPE, "M = %lld outside the launch contract 1 <= M <= 2^24", (long long)M);
  if (N < 64 || N > (1ll << 19))
    return fail(BSG_ERR_UNSUPPORTED_SHAPE, "N = %lld outside the launch contract 64 <= N <= 2^19", (long long)N);
  if (N % 8 != 0)
    return fail(BSG_ERR_ALIGNMENT, "N = %lld must be a multiple of 8 (16-byte BF16 output rows)", (long long)N);
  if (K > (1ll << 20)) return fail(BSG_ERR_UNSUPPORTED_SHAPE, "K = %lld above 2^20", (long long)K);
  if (!aligned(C, 16)) return fail(BSG_ERR_ALIGNMENT, "C must be 16-byte aligned");
  if (m_indices && !aligned(m_indices, 4)) return fail(BSG_ERR_ALIGNMENT, "m_indices must be 4-byte aligned");
  return BSG_OK;
}


// One GEMM launch through cudaLaunchKernelEx.  A grid smaller than the GPU (a small problem) is
// launched as a programmatic dependent of the previous kernel on the stream: its CTAs start on the
// idle SMs and do their set-up (barriers, TMEM, descriptor prefetch) while that kernel finishes, and
// wait for it on the device before touching memory (the FP8 page's M=65 shape: 5.5 -> 4.5 us per
// launch under graph replay).  Full-GPU grids keep plain stream order.  `pair`: 2-CTA clusters.
template <typename Kern, typename Params>
cudaError_t launch_gemm(Kern kernel, int grid, int threads, size_t smem, cudaStream_t cs, bool pair,
                        int sm_count, const Params& p) {
  cudaLaunchConfig_t lc = {};
  cudaLaunchAttribute la[2];
  int n = 0;
  if (grid < sm_count) {
    la[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    la[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (pair) {
    la[n].id = cudaLaunchAttributeClusterDimension;
    la[n].val.clusterDim.x = 2;
    la[n].val.clusterDim.y = 1;
    la[n].val.clusterDim.z = 1;
    ++n;
  }
  lc.gridDim = dim3(grid, 1, 1);
  lc.blockDim = dim3(threads, 1, 1);
  lc.dynamicSmemBytes = smem;
  lc.stream = cs;
  lc.attrs = la;
  lc.numAttrs = n;
  return cudaLaunchKernelEx(&lc, kernel, p);
}

// Raster groups of N tiles: when one expert's B (N x K bytes) fits comfortably in L2 the units run
// window-major (all N tiles of a window together); otherwise N tiles are grouped so that the group's
// slice of B (about 24 MB) stays resident while every window streams past it.
int n_group_for(int64_t N, int64_t row_bytes, int bn) {
  const int64_t n_tiles = (N + bn - 1) / bn;
  const int64_t b_bytes = N * row_bytes;
  if (b_bytes <= (48ll << 20)) return static_cast<int>(n_tiles);
  int64_t g = (24ll << 20) / (static_cast<int64_t>(bn) * row_bytes);
  if (g < 1) g = 1;
  return static_cast<int>(g < n_tiles ? g : n_tiles);
}

int grid_for(int sm_count, int64_t M, int64_t N, int64_t G, int bn) {
  const int64_t n_tiles = (N + bn - 1) / bn;
  const int64_t windows = (M + 127) / 128;
  const int64_t segs = windows + (G < M ? G : M);  // sorted routing: at most one extra segment per expert
  const int64_t units = n_tiles * segs;
  return static_cast<int>(units < sm_count ? units : sm_count);
}

}  // namespace


extern "C" {

const char* bsg_version(void) { return BSG_VERSION_STRING; }

const char* bsg_last_error(void) { return g_last_error.c_str(); }

uint64_t bsg_set_wait_timeout_ns(uint64_t ns) {
  std::lock_guard<std::mutex> lock(g_mu);
  uint64_t prev = g_timeout_ns;
  g_timeout_ns = ns ? ns : 2000000000ull;
  return prev;
}

static uint64_t current_timeout() {
  std::lock_guard<std::mutex> lock(g_mu);
  return g_timeout_ns;
}

static int current_fault() {
  std::lock_guard<std::mutex> lock(g_mu);
  return g_debug_fault;
}

bsg_status bsg_debug_set_fault(int mode) {
  if (mode < 0 || mode > bsg::kDebugWithholdSchedule) return fail(BSG_ERR_INVALID_ARG, "unknown fault mode %d", mode);
  std::lock_guard<std::mutex> lock(g_mu);
  g_debug_fault = mode;
  return BSG_OK;
}

}  // extern "C"

namespace {

bsg_status fp8_check(const void* A, const void* B, const float* a_scale, const float* b_scale,
                     const int32_t* m_indices, const void* C, int64_t M, int64_t N, int64_t K, int64_t G,
                     DeviceState** dev_out) {
  bsg_status st = check_common(A, B, m_indices, C, M, N, K, G);
  if (st != BSG_OK) return st;
  if (!a_scale || !b_scale) return fail(BSG_ERR_INVALID_ARG, "a_scale and b_scale must be non-null");
  if (K < 128 || K % 128 != 0)
    return fail(BSG_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 128 (one FP32 scale per 128)",
                (long long)K);
  if (!aligned(A, 16) || !aligned(B, 16)) return fail(BSG_ERR_ALIGNMENT, "A and B must be 16-byte aligned");
  if (!aligned(a_scale, 4) || !aligned(b_scale, 4))
    return fail(BSG_ERR_ALIGNMENT, "a_scale and b_scale must be 4-byte aligned");
  return device_state(dev_out);
}

// tactics 2 and 3: the operand-swapped kernel for experts with few rows; 128 (tactic 2) or 256
// (tactic 3) output columns per unit, token chunks of at most 128 / 64 rows
bsg_status fp8_swap_launch(DeviceState* dev, const void* A, const void* B, const float* a_scale,
                           const float* b_scale, const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K,
                           int64_t G, bsg_stream_t stream, int tactic) {
  bsg_status st;
  const int nh = tactic == 3 ? 2 : 1;
  const int bnr = 128 * nh;
  bsg::Fp8Params p;
  memset(&p, 0, sizeof(p));
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t str[1] = {static_cast<uint64_t>(K)};
    const uint32_t box[2] = {128u, static_cast<uint32_t>(bsg::fp8s::A_BOX)};
    const bool oob[2] = {false, true};  // a chunk's last box may run past M: zero-filled, never stored
    if ((st = encode(&p.tmA, "A", A, 2, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_128B)) != BSG_OK) return st;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), static_cast<uint64_t>(G)};
    const uint64_t str[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N) * static_cast<uint64_t>(K)};
    const uint32_t box[3] = {128u, static_cast<uint32_t>(bnr), 1u};
    const bool oob[3] = {false, true, false};
    if ((st = encode(&p.tmB, "B", B, 3, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_128B)) != BSG_OK) return st;
  }
  p.a_scale = a_scale;
  p.b_scale = b_scale;
  p.m_indices = m_indices;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = static_cast<int>(G);
  // few windows: N tile outermost, so consecutive chunks of one expert (a run crossing a window
  // boundary) read the same B tile at the same time; otherwise the usual raster groups
  const int64_t windows = (M + 127) / 128;
  p.n_group = windows <= 32 ? 1 : n_group_for(N, K, bnr);
  p.timeout_ns = current_timeout();
  p.status = dev->status;
  p.debug_mode = current_fault();

  cudaError_t e;
  if (!dev->fp8_swap_attr) {
    e = cudaFuncSetAttribute(bsg::fp8s::bsg_fp8_swap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bsg::fp8s::smem_bytes<1>()));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fp8 swapped kernel smem)");
    e = cudaFuncSetAttribute(bsg::fp8s::bsg_fp8_swap_n256_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bsg::fp8s::smem_bytes<2>()));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fp8 swapped 256-column kernel smem)");
    dev->fp8_swap_attr = true;
  }
  // units: chunks x N tiles; sorted routing gives at most windows + min(G, M) segments, each cut into
  // at most 128 / TM chunks
  const int64_t n_tiles = (N + bnr - 1) / bnr;
  const int64_t chunks = (windows + (G < M ? G : M)) * nh;
  const int64_t units = n_tiles * chunks;
  const int grid = bsg_forced_grid(0, static_cast<int>(units < dev->sm_count ? units : dev->sm_count));
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (nh == 1)
    e = launch_gemm(bsg::fp8s::bsg_fp8_swap_kernel, grid, bsg::fp8s::THREADS, bsg::fp8s::smem_bytes<1>(), cs, false,
                    dev->sm_count, p);
  else
    e = launch_gemm(bsg::fp8s::bsg_fp8_swap_n256_kernel, grid, bsg::fp8s::THREADS, bsg::fp8s::smem_bytes<2>(), cs,
                    false, dev->sm_count, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the fp8 swapped kernel");
  return BSG_OK;
}

// tactic 0: one SM per 128 x 256 tile; tactic 1: an SM pair per 256 x 256 tile (cta_group::2);
// tactics 2, 3: fp8_swap_launch; tactic 4: one SM per 128 x 64 tile (small problems)
bsg_status fp8_launch(DeviceState* dev, const void* A, const void* B, const float* a_scale, const float* b_scale,
                      const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G,
                      bsg_stream_t stream, int tactic) {
  if (tactic == 2 || tactic == 3)
    return fp8_swap_launch(dev, A, B, a_scale, b_scale, m_indices, C, M, N, K, G, stream, tactic);
  bsg_status st;
  const int cg = tactic == 1 ? 2 : 1;
  const bool n64 = tactic == 4;

  bsg::Fp8Params p;
  memset(&p, 0, sizeof(p));
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
    const uint64_t str[1] = {static_cast<uint64_t>(K)};
    const uint32_t box[2] = {128u, 128u};
    const bool oob[2] = {false, true};  // the last window may run past M: zero-filled, rows masked
    if ((st = encode(&p.tmA, "A", A, 2, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_128B)) != BSG_OK) return st;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), static_cast<uint64_t>(G)};
    const uint64_t str[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N) * static_cast<uint64_t>(K)};
    // B rows per CTA and stage: 256 (one SM, 256-column tile), 128 (each CTA of an SM pair, half of
    // the pair's 256-column tile) or 64 (the 64-column tile)
    const uint32_t box[3] = {128u,
                             static_cast<uint32_t>(n64       ? bsg::fp8::Cfg<1, 64>::B_BOX_ROWS
                                                   : cg == 2 ? bsg::fp8::Cfg<2>::B_BOX_ROWS
                                                             : bsg::fp8::Cfg<1>::B_BOX_ROWS),
                             1u};
    const bool oob[3] = {false, true, false};  // an N tail tile is zero-filled, columns masked
    if ((st = encode(&p.tmB, "B", B, 3, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_128B)) != BSG_OK) return st;
  }
  p.a_scale = a_scale;
  p.b_scale = b_scale;
  p.m_indices = m_indices;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = static_cast<int>(G);
  const int bn = n64 ? 64 : (cg == 2 ? bsg::fp8::Cfg<2>::BN : bsg::fp8::Cfg<1>::BN);
  p.n_group = n_group_for(N, K, bn);
  p.timeout_ns = current_timeout();
  p.status = dev->status;
  p.debug_mode = current_fault();

  cudaError_t e;
  if (!dev->fp8_attr) {
    e = cudaFuncSetAttribute(bsg::fp8::bsg_fp8_grouped_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bsg::fp8::smem_bytes<1>()));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fp8 kernel smem)");
    e = cudaFuncSetAttribute(bsg::fp8::bsg_fp8_grouped_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bsg::fp8::smem_bytes<2>()));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fp8 2-SM kernel smem)");
    // how many SM-pair clusters can be resident at once
    cudaLaunchConfig_t qc = {};
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    qc.gridDim = dim3(2 * (dev->sm_count / 2), 1, 1);
    qc.blockDim = dim3(bsg::fp8::THREADS, 1, 1);
    qc.dynamicSmemBytes = bsg::fp8::smem_bytes<2>();
    qc.attrs = qa;
    qc.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, bsg::fp8::bsg_fp8_grouped_2sm_kernel, &qc);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(fp8 2-SM kernel)");
    dev->fp8_pair_clusters = clusters;
    dev->fp8_attr = true;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (n64) {
    if (!dev->fp8_n64_attr) {
      e = cudaFuncSetAttribute(bsg::fp8::bsg_fp8_grouped_n64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(bsg::fp8::smem_bytes<1, 64>()));
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(fp8 64-column kernel smem)");
      dev->fp8_n64_attr = true;
    }
    const int grid = bsg_forced_grid(0, grid_for(dev->sm_count, M, N, G, bn));
    e = launch_gemm(bsg::fp8::bsg_fp8_grouped_n64_kernel, grid, bsg::fp8::THREADS, bsg::fp8::smem_bytes<1, 64>(), cs,
                    false, dev->sm_count, p);
  } else if (cg == 1) {
    const int grid = bsg_forced_grid(0, grid_for(dev->sm_count, M, N, G, bn));
    e = launch_gemm(bsg::fp8::bsg_fp8_grouped_kernel, grid, bsg::fp8::THREADS, bsg::fp8::smem_bytes<1>(), cs, false,
                    dev->sm_count, p);
  } else {
    if (dev->fp8_pair_clusters < 1) return fail(BSG_ERR_CUDA, "no SM-pair cluster fits on this device");
    const BsgUnitEstimate est = bsg_estimate_units(M, G);
    const int64_t n_tiles = (N + bn - 1) / bn;
    int64_t clusters = est.pairs_max * n_tiles;
    if (clusters > dev->fp8_pair_clusters) clusters = dev->fp8_pair_clusters;
    const int grid = 2 * ((bsg_forced_grid(0, static_cast<int>(2 * clusters)) + 1) / 2);
    e = launch_gemm(bsg::fp8::bsg_fp8_grouped_2sm_kernel, grid, bsg::fp8::THREADS, bsg::fp8::smem_bytes<2>(), cs, true,
                    dev->sm_count, p);
    if (e != cudaSuccess) return cuda_fail(e, "launch of the fp8 2-SM grouped kernel");
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the fp8 grouped kernel");
  return BSG_OK;
}

bsg_status nvfp4_check(const void* A, const void* B, const void* sfa, const void* sfb, const float* alpha,
                       const int32_t* m_indices, const void* C, int64_t M, int64_t N, int64_t K, int64_t G,
                       DeviceState** dev_out) {
  bsg_status st = check_common(A, B, m_indices, C, M, N, K, G);
  if (st != BSG_OK) return st;
  if (!sfa || !sfb || !alpha) return fail(BSG_ERR_INVALID_ARG, "sfa, sfb and alpha must be non-null");
  if (K < 256 || K % 256 != 0)
    return fail(BSG_ERR_UNSUPPORTED_SHAPE,
                "K = %lld must be a positive multiple of 256 (16-byte rows of packed codes and of scale bytes)",
                (long long)K);
  if (!aligned(alpha, 4)) return fail(BSG_ERR_ALIGNMENT, "alpha must be 4-byte aligned");
  return device_state(dev_out);
}

// tactic 0: one SM per 128 x 256 tile; tactic 1: an SM pair per 256 x 256 tile (cta_group::2)
bsg_status nvfp4_launch(DeviceState* dev, const void* A, const void* B, const void* sfa, const void* sfb,
                        const float* alpha, const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K,
                        int64_t G, bsg_stream_t stream, int tactic) {
  bsg_status st;
  const int cg = tactic == 1 ? 2 : 1;

  bsg::Nvfp4Params p;
  memset(&p, 0, sizeof(p));
  const uint64_t Kb = static_cast<uint64_t>(K) / 2;   // packed bytes per row
  const uint64_t Ks = static_cast<uint64_t>(K) / 16;  // scale bytes per row
  {
    const uint64_t dims[2] = {Kb, static_cast<uint64_t>(M)};
    const uint64_t str[1] = {Kb};
    const uint32_t box[2] = {128u, 128u};
    const bool oob[2] = {false, true};
    if ((st = encode(&p.tmA, "A", A, 2, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_128B)) != BSG_OK) return st;
  }
  {
    const uint64_t dims[3] = {Kb, static_cast<uint64_t>(N), static_cast<uint64_t>(G)};
    const uint64_t str[2] = {Kb, static_cast<uint64_t>(N) * Kb};
    // B rows per CTA and stage: 256 (one SM) or 128 (each CTA of an SM pair)
    const uint32_t box[3] = {128u, static_cast<uint32_t>(bsg::nvfp4::BN / cg), 1u};
    const bool oob[3] = {false, true, false};
    if ((st = encode(&p.tmB, "B", B, 3, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_128B)) != BSG_OK) return st;
  }
  {
    const uint64_t dims[2] = {Ks, static_cast<uint64_t>(M)};
    const uint64_t str[1] = {Ks};
    const uint32_t box[2] = {16u, 128u};
    const bool oob[2] = {false, true};
    if ((st = encode(&p.tmSFA, "sfa", sfa, 2, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_NONE)) != BSG_OK) return st;
  }
  {
    const uint64_t dims[3] = {Ks, static_cast<uint64_t>(N), static_cast<uint64_t>(G)};
    const uint64_t str[2] = {Ks, static_cast<uint64_t>(N) * Ks};
    const uint32_t box[3] = {16u, static_cast<uint32_t>(bsg::nvfp4::BN), 1u};
    const bool oob[3] = {false, true, false};
    if ((st = encode(&p.tmSFB, "sfb", sfb, 3, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_NONE)) != BSG_OK) return st;
  }
  {
    const uint64_t dims[2] = {2 * static_cast<uint64_t>(N), static_cast<uint64_t>(M)};
    const uint64_t str[1] = {2 * static_cast<uint64_t>(N)};
    const uint32_t box[2] = {128u, 32u};
    const bool oob[2] = {true, true};
    if ((st = encode(&p.tmC, "C", C, 2, dims, str, box, oob, CU_TENSOR_MAP_SWIZZLE_128B)) != BSG_OK) return st;
  }
  p.alpha = alpha;
  p.m_indices = m_indices;
  p.C = static_cast<__nv_bfloat16*>(C);
  p.M = static_cast<int>(M);
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.G = static_cast<int>(G);
  p.n_group = n_group_for(N, K / 2 + K / 16, bsg::nvfp4::BN);
  p.timeout_ns = current_timeout();
  p.status = dev->status;
  p.debug_mode = current_fault();

  cudaError_t e;
  if (!dev->nvfp4_attr) {
    e = cudaFuncSetAttribute(bsg::nvfp4::bsg_nvfp4_grouped_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bsg::nvfp4::smem_bytes<1>()));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(nvfp4 kernel smem)");
    e = cudaFuncSetAttribute(bsg::nvfp4::bsg_nvfp4_grouped_2sm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(bsg::nvfp4::smem_bytes<2>()));
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(nvfp4 2-SM kernel smem)");
    cudaLaunchConfig_t qc = {};
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 2;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    qc.gridDim = dim3(2 * (dev->sm_count / 2), 1, 1);
    qc.blockDim = dim3(bsg::nvfp4::THREADS, 1, 1);
    qc.dynamicSmemBytes = bsg::nvfp4::smem_bytes<2>();
    qc.attrs = qa;
    qc.numAttrs = 1;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, bsg::nvfp4::bsg_nvfp4_grouped_2sm_kernel, &qc);
    if (e != cudaSuccess) return cuda_fail(e, "cudaOccupancyMaxActiveClusters(nvfp4 2-SM kernel)");
    dev->nvfp4_pair_clusters = clusters;
    dev->nvfp4_attr = true;
  }
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (cg == 1) {
    const int grid = bsg_forced_grid(1, grid_for(dev->sm_count, M, N, G, bsg::nvfp4::BN));
    e = launch_gemm(bsg::nvfp4::bsg_nvfp4_grouped_kernel, grid, bsg::nvfp4::THREADS, bsg::nvfp4::smem_bytes<1>(), cs,
                    false, dev->sm_count, p);
  } else {
    if (dev->nvfp4_pair_clusters < 1) return fail(BSG_ERR_CUDA, "no SM-pair cluster fits on this device");
    const BsgUnitEstimate est = bsg_estimate_units(M, G);
    const int64_t n_tiles = (N + bsg::nvfp4::BN - 1) / bsg::nvfp4::BN;
    int64_t clusters = est.pairs_max * n_tiles;
    if (clusters > dev->nvfp4_pair_clusters) clusters = dev->nvfp4_pair_clusters;
    const int grid = 2 * ((bsg_forced_grid(1, static_cast<int>(2 * clusters)) + 1) / 2);
    e = launch_gemm(bsg::nvfp4::bsg_nvfp4_grouped_2sm_kernel, grid, bsg::nvfp4::THREADS, bsg::nvfp4::smem_bytes<2>(),
                    cs, true, dev->sm_count, p);
    if (e != cudaSuccess) return cuda_fail(e, "launch of the nvfp4 2-SM kernel");
  }
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the nvfp4 kernel");
  return BSG_OK;
}

// Times `reps` launches of every tactic (after one warm-up launch each) with CUDA events on the
// stream; returns the fastest tactic or a negative status.  `launch(t)` enqueues one call.  A tactic
// whose launches gave up a bounded wait returned early and would look fastest: the device status
// word is read (not cleared, so bsg_get_device_status still reports it) after each tactic, and a set
// word ends the tuning with BSG_ERR_DEVICE_TIMEOUT and records nothing.
template <typename Launch>
int time_tactics(DeviceState* dev, int kind, int reps, bsg_stream_t stream, Launch launch) {
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  cudaEvent_t ev[2];
  if (cudaEventCreate(&ev[0]) != cudaSuccess) return cuda_fail(cudaGetLastError(), "cudaEventCreate");
  if (cudaEventCreate(&ev[1]) != cudaSuccess) {
    cudaEventDestroy(ev[0]);
    return cuda_fail(cudaGetLastError(), "cudaEventCreate");
  }
  int best = BSG_ERR_CUDA;
  float best_ms = 0.f;
  const int n = bsg_num_tactics(kind);
  bsg_status st = BSG_OK;
  for (int t = 0; t < n && st == BSG_OK; ++t) {
    if ((st = launch(t)) != BSG_OK) break;
    cudaEventRecord(ev[0], cs);
    for (int r = 0; r < reps && st == BSG_OK; ++r) st = launch(t);
    cudaEventRecord(ev[1], cs);
    cudaError_t e = cudaEventSynchronize(ev[1]);
    if (st != BSG_OK) break;
    if (e != cudaSuccess) {
      st = cuda_fail(e, "timing a tactic");
      break;
    }
    bsg::DeviceStatus hs = {0u, 0u};
    e = cudaMemcpy(&hs, dev->status, sizeof(hs), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) {
      st = cuda_fail(e, "reading the device status word");
      break;
    }
    if (hs.word != 0u) {
      st = fail(BSG_ERR_DEVICE_TIMEOUT,
                "tactic %d (%s) gave up a bounded wait while being timed (status word 0x%08x); nothing recorded",
                t, bsg_tactic_name(kind, t), hs.word);
      break;
    }
    float ms = 0.f;
    cudaEventElapsedTime(&ms, ev[0], ev[1]);
    if (best < 0 || ms < best_ms) {
      best = t;
      best_ms = ms;
    }
  }
  cudaEventDestroy(ev[0]);
  cudaEventDestroy(ev[1]);
  return st != BSG_OK ? static_cast<int>(st) : best;
}

}  // namespace

extern "C" {

bsg_status bsg_fp8_grouped_gemm(const void* A, const void* B, const float* a_scale, const float* b_scale,
                                const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G,
                                bsg_stream_t stream) {
  g_last_error.clear();
  DeviceState* dev = nullptr;
  bsg_status st = fp8_check(A, B, a_scale, b_scale, m_indices, C, M, N, K, G, &dev);
  if (st != BSG_OK) return st;
  const int tactic = bsg_choose_tactic(0, M, N, K, G, dev->sm_count);
  return fp8_launch(dev, A, B, a_scale, b_scale, m_indices, C, M, N, K, G, stream, tactic);
}

bsg_status bsg_nvfp4_gemm(const void* A, const void* B, const void* sfa, const void* sfb, const float* alpha,
                          const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G,
                          bsg_stream_t stream) {
  g_last_error.clear();
  DeviceState* dev = nullptr;
  bsg_status st = nvfp4_check(A, B, sfa, sfb, alpha, m_indices, C, M, N, K, G, &dev);
  if (st != BSG_OK) return st;
  const int tactic = bsg_choose_tactic(1, M, N, K, G, dev->sm_count);
  return nvfp4_launch(dev, A, B, sfa, sfb, alpha, m_indices, C, M, N, K, G, stream, tactic);
}

int bsg_autotune_fp8(const void* A, const void* B, const float* a_scale, const float* b_scale,
                     const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G, int reps,
                     bsg_stream_t stream) {
  g_last_error.clear();
  if (reps < 1 || reps > 10000) return fail(BSG_ERR_INVALID_ARG, "reps = %d outside [1, 10000]", reps);
  DeviceState* dev = nullptr;
  bsg_status st = fp8_check(A, B, a_scale, b_scale, m_indices, C, M, N, K, G, &dev);
  if (st != BSG_OK) return st;
  const int best = time_tactics(dev, 0, reps, stream, [&](int t) {
    return fp8_launch(dev, A, B, a_scale, b_scale, m_indices, C, M, N, K, G, stream, t);
  });
  if (best >= 0) bsg_record_tuned(0, M, N, K, G, best);
  return best;
}

int bsg_autotune_nvfp4(const void* A, const void* B, const void* sfa, const void* sfb, const float* alpha,
                       const int32_t* m_indices, void* C, int64_t M, int64_t N, int64_t K, int64_t G, int reps,
                       bsg_stream_t stream) {
  g_last_error.clear();
  if (reps < 1 || reps > 10000) return fail(BSG_ERR_INVALID_ARG, "reps = %d outside [1, 10000]", reps);
  DeviceState* dev = nullptr;
  bsg_status st = nvfp4_check(A, B, sfa, sfb, alpha, m_indices, C, M, N, K, G, &dev);
  if (st != BSG_OK) return st;
  const int best = time_tactics(dev, 1, reps, stream, [&](int t) {
    return nvfp4_launch(dev, A, B, sfa, sfb, alpha, m_indices, C, M, N, K, G, stream, t);
  });
  if (best >= 0) bsg_record_tuned(1, M, N, K, G, best);
  return best;
}

static bsg_status check_quant(const void* X, const int32_t* src_rows, const void* A, const void* scale, int64_t M_in,
                              int64_t M, int64_t K, int64_t k_multiple) {
  if (!X || !A || !scale) return fail(BSG_ERR_INVALID_ARG, "X, A and the scale output must be non-null");
  if (M < 1 || M_in < 1 || M > 0x7FFFFFFFll || M_in > 0x7FFFFFFFll)
    return fail(BSG_ERR_UNSUPPORTED_SHAPE, "M = %lld and M_in = %lld must lie in [1, 2^31 - 1]", (long long)M,
                (long long)M_in);
  if (!src_rows && M > M_in)
    return fail(BSG_ERR_INVALID_ARG, "without src_rows every output row m reads input row m: M = %lld > M_in = %lld",
                (long long)M, (long long)M_in);
  if (K < 16 || K > (1ll << 20) || K % k_multiple != 0)
    return fail(BSG_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a multiple of %lld in [16, 2^20]", (long long)K,
                (long long)k_multiple);
  if (!aligned(X, 16) || !aligned(A, 16)) return fail(BSG_ERR_ALIGNMENT, "X and A must be 16-byte aligned");
  if (src_rows && !aligned(src_rows, 4)) return fail(BSG_ERR_ALIGNMENT, "src_rows must be 4-byte aligned");
  return BSG_OK;
}

static int quant_grid(int sm_count, int64_t M, int64_t K, int64_t cols_per_task) {
  const int64_t tasks = M * ((K + cols_per_task - 1) / cols_per_task);            // one warp each
  const int64_t blocks = (tasks + bsg::quant::THREADS / 32 - 1) / (bsg::quant::THREADS / 32);
  const int64_t cap = static_cast<int64_t>(sm_count) * (2048 / bsg::quant::THREADS);
  return static_cast<int>(blocks < cap ? blocks : cap);
}

bsg_status bsg_quantize_fp8_rows(const void* X, const int32_t* src_rows, void* A, float* a_scale, int64_t M_in,
                                 int64_t M, int64_t K, bsg_stream_t stream) {
  g_last_error.clear();
  bsg_status st = check_quant(X, src_rows, A, a_scale, M_in, M, K, 128);
  if (st != BSG_OK) return st;
  if (!aligned(a_scale, 4)) return fail(BSG_ERR_ALIGNMENT, "a_scale must be 4-byte aligned");
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != BSG_OK) return st;
  bsg::quant::QuantParams p;
  memset(&p, 0, sizeof(p));
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.src_rows = src_rows;
  p.A = static_cast<uint8_t*>(A);
  p.scale = a_scale;
  p.M_in = M_in;
  p.M = M;
  p.K = static_cast<int>(K);
  bsg::quant::bsg_quant_fp8_rows_kernel<<<quant_grid(dev->sm_count, M, K, bsg::quant::CHUNK * bsg::quant::GROUP), bsg::quant::THREADS, 0,
                                          reinterpret_cast<cudaStream_t>(stream)>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the fp8 quantisation kernel");
  return BSG_OK;
}

bsg_status bsg_quantize_nvfp4_rows(const void* X, const int32_t* src_rows, const float* global_scale, void* A,
                                   void* sfa, int64_t M_in, int64_t M, int64_t K, bsg_stream_t stream) {
  g_last_error.clear();
  bsg_status st = check_quant(X, src_rows, A, sfa, M_in, M, K, 16);
  if (st != BSG_OK) return st;
  if (!global_scale || !aligned(global_scale, 4))
    return fail(BSG_ERR_INVALID_ARG, "global_scale must be a non-null, 4-byte aligned device pointer");
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != BSG_OK) return st;
  bsg::quant::QuantParams p;
  memset(&p, 0, sizeof(p));
  p.X = static_cast<const __nv_bfloat16*>(X);
  p.src_rows = src_rows;
  p.gs = global_scale;
  p.A = static_cast<uint8_t*>(A);
  p.scale = sfa;
  p.M_in = M_in;
  p.M = M;
  p.K = static_cast<int>(K);
  bsg::quant::bsg_quant_nvfp4_rows_kernel<<<quant_grid(dev->sm_count, M, K, bsg::quant::NV_CHUNK * bsg::quant::NV_GROUP), bsg::quant::THREADS, 0,
                                            reinterpret_cast<cudaStream_t>(stream)>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the nvfp4 quantisation kernel");
  return BSG_OK;
}

}  // extern "C"

namespace {

// Tiling of the MoE permutation: tiles of at least MIN_TILE entries (multiples of 32), at most
// cap_ints / G of them, so that the scratch (tiles x G int32 counters) stays within cap_ints.
struct MoePlan {
  bool fused = false;   // the single-CTA kernel (no scratch)
  int tile = 0;
  int tiles = 0;
  size_t scratch_bytes = 0;
};

constexpr int64_t kMoeWorkspaceCapInts = 1ll << 22;  // 16 MiB of counters at most

MoePlan moe_plan(int64_t n, int64_t G, int64_t cap_ints) {
  MoePlan pl;
  if (n <= bsg::moe::FUSED_MAX_N && G <= bsg::moe::FUSED_MAX_G) {
    const int64_t per = (n + bsg::moe::FUSED_WARPS - 1) / bsg::moe::FUSED_WARPS;
    pl.fused = true;
    pl.tile = static_cast<int>((per + 31) / 32 * 32);
    pl.tiles = bsg::moe::FUSED_WARPS;
    return pl;
  }
  int64_t tiles = (n + bsg::moe::MIN_TILE - 1) / bsg::moe::MIN_TILE;
  if (tiles < 1) tiles = 1;
  if (tiles > bsg::moe::MAX_TILES) tiles = bsg::moe::MAX_TILES;
  if (tiles * G > cap_ints) tiles = cap_ints / G > 1 ? cap_ints / G : 1;
  int64_t tile = (n + tiles - 1) / tiles;
  tile = (tile + 31) / 32 * 32;
  tiles = (n + tile - 1) / tile;
  pl.tile = static_cast<int>(tile);
  pl.tiles = static_cast<int>(tiles);
  pl.scratch_bytes = static_cast<size_t>(tiles) * static_cast<size_t>(G) * sizeof(int32_t);
  return pl;
}

bsg_status moe_check_sizes(int64_t T, int64_t top_k, int64_t G) {
  if (T < 1 || top_k < 1 || top_k > 256)
    return fail(BSG_ERR_UNSUPPORTED_SHAPE, "T = %lld and top_k = %lld must satisfy T >= 1, 1 <= top_k <= 256",
                (long long)T, (long long)top_k);
  if (T * top_k > (1ll << 24))
    return fail(BSG_ERR_UNSUPPORTED_SHAPE, "T * top_k = %lld above 2^24 (the grouped GEMM's row limit)",
                (long long)(T * top_k));
  if (G < 1 || G > 4096) return fail(BSG_ERR_UNSUPPORTED_SHAPE, "G = %lld outside [1, 4096]", (long long)G);
  return BSG_OK;
}

bsg_status moe_check(const int32_t* expert_ids, int64_t T, int64_t top_k, int64_t G, const int32_t* src_rows,
                     const int32_t* m_indices, const int32_t* dst_rows, const int32_t* expert_offsets) {
  bsg_status st = moe_check_sizes(T, top_k, G);
  if (st != BSG_OK) return st;
  if (!expert_ids || !src_rows || !m_indices || !dst_rows || !expert_offsets)
    return fail(BSG_ERR_INVALID_ARG, "expert_ids, src_rows, m_indices, dst_rows and expert_offsets must be non-null");
  if (!aligned(expert_ids, 4) || !aligned(src_rows, 4) || !aligned(m_indices, 4) || !aligned(dst_rows, 4) ||
      !aligned(expert_offsets, 4))
    return fail(BSG_ERR_ALIGNMENT, "the MoE permutation's int32 arrays must be 4-byte aligned");
  return BSG_OK;
}

// The permutation on `stream`: the single-CTA kernel, or the three kernels with `scratch`
// (pl.scratch_bytes, 4-byte aligned).
bsg_status moe_launch(DeviceState* dev, const int32_t* expert_ids, int64_t T, int64_t top_k, int64_t G,
                      int32_t* src_rows, int32_t* m_indices, int32_t* dst_rows, int32_t* expert_offsets,
                      int32_t* scratch, const MoePlan& pl, bsg_stream_t stream) {
  cudaError_t e;
  if (!dev->moe_attr) {
    const int smem = bsg::moe::WARPS * 4096 * static_cast<int>(sizeof(int32_t));
    e = cudaFuncSetAttribute(bsg::moe::bsg_moe_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(moe count kernel smem)");
    e = cudaFuncSetAttribute(bsg::moe::bsg_moe_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(moe scatter kernel smem)");
    const int fused_smem = bsg::moe::FUSED_WARPS * bsg::moe::FUSED_MAX_G * static_cast<int>(sizeof(int32_t));
    e = cudaFuncSetAttribute(bsg::moe::bsg_moe_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, fused_smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(moe single-CTA kernel smem)");
    dev->moe_attr = true;
  }
  bsg::moe::Params p;
  memset(&p, 0, sizeof(p));
  p.expert_ids = expert_ids;
  p.src_rows = src_rows;
  p.m_indices = m_indices;
  p.dst_rows = dst_rows;
  p.expert_offsets = expert_offsets;
  p.scratch = scratch;
  p.n = T * top_k;
  p.top_k = static_cast<int>(top_k);
  p.G = static_cast<int>(G);
  p.tile = pl.tile;
  p.tiles = pl.tiles;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (pl.fused) {
    const size_t smem = static_cast<size_t>(bsg::moe::FUSED_WARPS) * static_cast<size_t>(G) * sizeof(int32_t);
    bsg::moe::bsg_moe_fused_kernel<<<1, bsg::moe::FUSED_THREADS, smem, cs>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "launch of the MoE permutation kernel");
    return BSG_OK;
  }
  const int blocks = (pl.tiles + bsg::moe::WARPS - 1) / bsg::moe::WARPS;
  const size_t tile_smem = static_cast<size_t>(bsg::moe::WARPS) * static_cast<size_t>(G) * sizeof(int32_t);
  bsg::moe::bsg_moe_count_kernel<<<blocks, bsg::moe::THREADS, tile_smem, cs>>>(p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "launch of the MoE count kernel");
  const int64_t scan_segments = G <= bsg::moe::SCAN_THREADS ? bsg::moe::SCAN_THREADS / G : 1;
  const size_t scan_smem = static_cast<size_t>(scan_segments * G + G) * sizeof(int32_t);   // <= 32 KiB
  // the scan and scatter kernels start their launch while the previous kernel runs and wait for it
  // on the device (programmatic dependent launch)
  cudaLaunchAttribute la[1];
  la[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  la[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t lc = {};
  lc.stream = cs;
  lc.attrs = la;
  lc.numAttrs = 1;
  lc.gridDim = dim3(1, 1, 1);
  lc.blockDim = dim3(bsg::moe::SCAN_THREADS, 1, 1);
  lc.dynamicSmemBytes = scan_smem;
  e = cudaLaunchKernelEx(&lc, bsg::moe::bsg_moe_scan_kernel, p);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the MoE scan kernel");
  lc.gridDim = dim3(blocks, 1, 1);
  lc.blockDim = dim3(bsg::moe::THREADS, 1, 1);
  lc.dynamicSmemBytes = tile_smem;
  e = cudaLaunchKernelEx(&lc, bsg::moe::bsg_moe_scatter_kernel, p);
  if (e != cudaSuccess) return cuda_fail(e, "launch of the MoE scatter kernel");
  return BSG_OK;
}

}  // namespace

extern "C" {

bsg_status bsg_moe_permute_workspace_size(int64_t T, int64_t top_k, int64_t G, size_t* bytes) {
  g_last_error.clear();
  if (!bytes) return fail(BSG_ERR_INVALID_ARG, "bytes must be non-null");
  bsg_status st = moe_check_sizes(T, top_k, G);
  if (st != BSG_OK) return st;
  *bytes = moe_plan(T * top_k, G, kMoeWorkspaceCapInts).scratch_bytes;
  return BSG_OK;
}

bsg_status bsg_moe_permute(const int32_t* expert_ids, int64_t T, int64_t top_k, int64_t G, int32_t* src_rows,
                           int32_t* m_indices, int32_t* dst_rows, int32_t* expert_offsets, void* workspace,
                           size_t workspace_bytes, bsg_stream_t stream) {
  g_last_error.clear();
  bsg_status st = moe_check(expert_ids, T, top_k, G, src_rows, m_indices, dst_rows, expert_offsets);
  if (st != BSG_OK) return st;
  const MoePlan pl = moe_plan(T * top_k, G, kMoeWorkspaceCapInts);
  if (pl.scratch_bytes > 0 && (!workspace || workspace_bytes < pl.scratch_bytes))
    return fail(BSG_ERR_INVALID_ARG, "workspace of %zu bytes is missing or smaller than the %zu bytes needed",
                workspace_bytes, pl.scratch_bytes);
  if (workspace && !aligned(workspace, 16)) return fail(BSG_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != BSG_OK) return st;
  return moe_launch(dev, expert_ids, T, top_k, G, src_rows, m_indices, dst_rows, expert_offsets,
                    static_cast<int32_t*>(workspace), pl, stream);
}

}  // extern "C"

namespace {

// Scratch of bsg_moe_permute_noalloc: one array in the library's device image (every GPU that loads
// the library holds it until the process exits), shared by every call on that GPU.  Host code sees
// only a host-side stand-in under this name, so the device address is looked up once per device.
constexpr size_t kMoeStaticScratchBytes = 2u << 20;   // 2 MiB = 524288 int32 counters
static __device__ __align__(256) int32_t g_moe_static_scratch[kMoeStaticScratchBytes / sizeof(int32_t)];

int32_t* g_moe_static_addr[kMaxDevices] = {};

// The device address of the static scratch on the current device (looked up on the first call for
// that device, with that device current).
bsg_status moe_static_scratch(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(BSG_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_moe_static_addr[dev]) {
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_moe_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(MoE permutation scratch)");
    g_moe_static_addr[dev] = static_cast<int32_t*>(addr);
  }
  *out = g_moe_static_addr[dev];
  return BSG_OK;
}

}  // namespace

extern "C" {

bsg_status bsg_moe_permute_noalloc(const int32_t* expert_ids, int64_t T, int64_t top_k, int64_t G,
                                   int32_t* src_rows, int32_t* m_indices, int32_t* dst_rows,
                                   int32_t* expert_offsets, bsg_stream_t stream) {
  g_last_error.clear();
  bsg_status st = moe_check(expert_ids, T, top_k, G, src_rows, m_indices, dst_rows, expert_offsets);
  if (st != BSG_OK) return st;
  const MoePlan pl = moe_plan(T * top_k, G, kMoeWorkspaceCapInts);
  if (pl.scratch_bytes > kMoeStaticScratchBytes)
    return fail(BSG_ERR_UNSUPPORTED_SHAPE,
                "T = %lld, top_k = %lld, G = %lld need %zu bytes of scratch, more than the %zu bytes this "
                "allocation-free entry point holds; call bsg_moe_permute with a workspace instead",
                (long long)T, (long long)top_k, (long long)G, pl.scratch_bytes, kMoeStaticScratchBytes);
  DeviceState* dev = nullptr;
  if ((st = device_state(&dev)) != BSG_OK) return st;
  int32_t* scratch = nullptr;
  if ((st = moe_static_scratch(&scratch)) != BSG_OK) return st;
  return moe_launch(dev, expert_ids, T, top_k, G, src_rows, m_indices, dst_rows, expert_offsets, scratch, pl,
                    stream);
}

bsg_status bsg_get_device_status(bsg_stream_t stream) {
  g_last_error.clear();
  DeviceState* dev = nullptr;
  bsg_status st = device_state(&dev);
  if (st != BSG_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  bsg::DeviceStatus hs;
  e = cudaMemcpy(&hs, dev->status, sizeof(hs), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status word");
  if (hs.word == 0) return BSG_OK;
  bsg::DeviceStatus zero = {0u, 0u};
  e = cudaMemcpy(dev->status, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device status word");
  return fail(BSG_ERR_DEVICE_TIMEOUT,
              "a kernel gave up a bounded wait: site %u, stage %u, block %u, parity %u (status word 0x%08x)",
              (hs.word >> 20) & 0xFu, (hs.word >> 12) & 0xFFu, hs.word & 0xFFFu, hs.detail, hs.word);
}

}  // extern "C"
