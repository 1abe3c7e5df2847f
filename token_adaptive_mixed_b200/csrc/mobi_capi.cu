// mobi_capi.cu — the C ABI of libmobi (declared in include/mobi.h): argument
// validation, kernel dispatch, the per-device status word and host helpers.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/mobi.h"
#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

// Launchers defined in the kernel files.
cudaError_t launch_pack(const void* W, int64_t N, int64_t K, int S, uint32_t* codes, uint32_t* sz,
                        cudaStream_t stream, int num_sms, int bits, int G);
cudaError_t launch_route(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias, int S,
                         int32_t* k_t, int32_t* perm, int32_t* offsets, void* ws, cudaStream_t stream);
size_t route_ws_bytes(int64_t T, int64_t K, int S);
cudaError_t launch_route_mlp(const void* X, int64_t T, int64_t K, const float* W1, const float* b1, int64_t H,
                             const float* W2, const float* b2, int S, double thr, int32_t* k_t, int32_t* perm,
                             int32_t* offsets, void* ws, cudaStream_t stream, int sms);
size_t route_mlp_ws_bytes(int64_t T, int64_t K, int64_t H, int sms);
cudaError_t launch_decode(const void* X, int T, int64_t K, const int32_t* k_t, const uint32_t* codes,
                          const uint32_t* sz, int64_t N, int S, float* Y, void* ws, cudaStream_t stream,
                          DeviceStatus* st, int bits, int mask1);
size_t decode_ws_bytes(int64_t N, int64_t K);
cudaError_t launch_prefill(const void* X, int64_t T, int64_t K, const int32_t* k_t, const int32_t* perm,
                           const int32_t* offsets, const uint32_t* codes, const uint32_t* sz, int64_t N, int S,
                           float* Y, void* ws, cudaStream_t stream, DeviceStatus* st, int bits, int mask1);
size_t prefill_ws_bytes(int64_t T, int64_t N, int64_t K);

static thread_local char g_last_error[256];

cudaError_t note_error(const char* where, cudaError_t e) {
  if (e != cudaSuccess) snprintf(g_last_error, sizeof g_last_error, "%s: %s (%s)", where, cudaGetErrorName(e),
                                 cudaGetErrorString(e));
  return e;
}

void note_message(const char* msg) { snprintf(g_last_error, sizeof g_last_error, "%s", msg); }

// One status block per device, in the module's device memory.
__device__ DeviceStatus g_device_status;

constexpr int kMaxDevices = 64;
static std::mutex g_mu;
static DeviceStatus* g_status_ptr[kMaxDevices];
static int g_sms[kMaxDevices];
static std::atomic<uint64_t> g_wait_limit[kMaxDevices];

static int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return (d >= 0 && d < kMaxDevices) ? d : -1;
}

DeviceStatus* device_status(cudaError_t* err) {
  const int d = current_device();
  *err = cudaSuccess;
  if (d < 0) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_status_ptr[d]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_device_status);
    if (e != cudaSuccess) {
      *err = e;
      return nullptr;
    }
    g_status_ptr[d] = static_cast<DeviceStatus*>(p);
  }
  return g_status_ptr[d];
}

uint64_t wait_limit() {
  const int d = current_device();
  if (d < 0) return kDefaultWaitLimit;
  const uint64_t v = g_wait_limit[d].load();
  return v ? v : kDefaultWaitLimit;
}

int num_sms() {
  const int d = current_device();
  if (d < 0) return 148;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_sms[d]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || v <= 0) v = 148;
    g_sms[d] = v;
  }
  return g_sms[d];
}

// The attribute is set once per (kernel, device, size): later calls only look
// it up, which keeps a driver call out of every launch.
cudaError_t set_smem(const void* func, int bytes) {
  struct Entry { const void* func; int device; int bytes; };
  static Entry done[64];
  static int ndone = 0;
  const int d = current_device();
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < ndone; ++i)
      if (done[i].func == func && done[i].device == d && done[i].bytes >= bytes) return cudaSuccess;
  }
  const cudaError_t e = note_error("cudaFuncSetAttribute(max dynamic shared memory)",
                                   cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (ndone < 64) done[ndone++] = Entry{func, d, bytes};
  }
  return e;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Encoded maps are a pure function of their arguments: a small cache keeps
// the driver's encoder out of repeated calls on the same buffers.
struct TmapKey {
  const void* base;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  int rank, elem_bytes, swizzle;
  bool operator==(const TmapKey& o) const { return memcmp(this, &o, sizeof *this) == 0; }
};
static constexpr int kTmapCache = 64;
static TmapKey g_tmap_key[kTmapCache];
static CUtensorMap g_tmap_val[kTmapCache];
static int g_tmap_n = 0, g_tmap_next = 0;

// Tiled tensor map of rank 2 or 3: dims[0] innermost (elements), strides[i] the
// byte stride of dimension i + 1, box in elements.
static bool make_tmap(CUtensorMap* map, const void* base, int elem_bytes, int rank, const uint64_t* dims,
                      const uint64_t* strides, const uint32_t* box, int swizzle_bytes) {
  TmapKey key;
  memset(&key, 0, sizeof key);  // padding included, so memcmp compares only what is set
  key.base = base;
  key.rank = rank;
  key.elem_bytes = elem_bytes;
  key.swizzle = swizzle_bytes;
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
    if (i + 1 < rank) key.strides[i] = strides[i];
  }
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (int i = 0; i < g_tmap_n; ++i)
      if (g_tmap_key[i] == key) {
        *map = g_tmap_val[i];
        return true;
      }
  }
  auto fn = encode_fn();
  if (!fn) return false;
  CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32;
  cuuint64_t cdims[3], cstr[2];
  cuuint32_t cbox[3], estr[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    cdims[i] = dims[i];
    cbox[i] = box[i];
    if (i + 1 < rank) cstr[i] = strides[i];
  }
  CUresult r = fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), cdims, cstr, cbox, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                  : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                  : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                        : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    snprintf(g_last_error, sizeof g_last_error,
             "cuTensorMapEncodeTiled: CUresult %d (rank %d, dims %llu x %llu x %llu, box %u x %u x %u, swizzle %d)",
             (int)r, rank, (unsigned long long)dims[0], (unsigned long long)dims[1],
             (unsigned long long)(rank > 2 ? dims[2] : 1), box[0], box[1], rank > 2 ? box[2] : 1, swizzle_bytes);
  if (r == CUDA_SUCCESS) {
    std::lock_guard<std::mutex> lock(g_mu);
    g_tmap_key[g_tmap_next] = key;
    g_tmap_val[g_tmap_next] = *map;
    g_tmap_next = (g_tmap_next + 1) % kTmapCache;
    if (g_tmap_n < kTmapCache) ++g_tmap_n;
  }
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
  const uint64_t dims[2] = {cols, rows}, strides[1] = {row_stride_bytes};
  const uint32_t box[2] = {box_cols, box_rows};
  return make_tmap(map, base, elem_bytes, 2, dims, strides, box, swizzle_bytes);
}

}  // namespace mobi

using namespace mobi;

namespace {

constexpr int64_t kMaxDim = int64_t(1) << 28;
constexpr int64_t kMaxMlpHidden = 65536;  // scorer hidden width: grid.y of the hidden-layer kernel stays small

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

mobi_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return MOBI_OK;
  if (!g_last_error[0]) note_error("CUDA", e);
  (void)cudaGetLastError();  // clear a sticky launch error
  return MOBI_ERR_CUDA;
}

mobi_status check_matrix(int64_t N, int64_t K, int G, int S) {
  if (N < 0 || K < 0 || S < 1 || S > kMaxSlices) return MOBI_ERR_INVALID_ARG;
  if (G != 128) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (K % 128 != 0 || N % 16 != 0 || N > kMaxDim || K > kMaxDim) return MOBI_ERR_UNSUPPORTED_SHAPE;
  return MOBI_OK;
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

namespace mobi {
mobi_status status_of(cudaError_t e) { return cuda_status(e); }
void clear_message() { g_last_error[0] = 0; }
}  // namespace mobi

extern "C" {

const char* mobi_status_string(mobi_status st) {
  switch (st) {
    case MOBI_OK: return "MOBI_OK";
    case MOBI_ERR_INVALID_ARG: return "MOBI_ERR_INVALID_ARG";
    case MOBI_ERR_UNSUPPORTED_SHAPE: return "MOBI_ERR_UNSUPPORTED_SHAPE";
    case MOBI_ERR_MISALIGNED: return "MOBI_ERR_MISALIGNED";
    case MOBI_ERR_WORKSPACE: return "MOBI_ERR_WORKSPACE";
    case MOBI_ERR_CUDA: return "MOBI_ERR_CUDA";
    case MOBI_ERR_TIMEOUT: return "MOBI_ERR_TIMEOUT";
    case MOBI_ERR_IO: return "MOBI_ERR_IO";
  }
  return "MOBI_ERR_UNKNOWN";
}

const char* mobi_last_error(void) { return g_last_error; }

int mobi_version(void) { return 100; }

namespace {
// Width mode of S slices: 2 or 1 when every slice has that width, 3 when they
// differ; mask1 has bit s set when slice s is 1-bit. False for an invalid
// width or S.
bool width_mode(int S, const int* widths, int* mode, int* mask1) {
  if (S < 1 || S > mobi::kMaxSlices || !widths) return false;
  int m = 0, n1 = 0;
  for (int j = 0; j < S; ++j) {
    if (widths[j] != 1 && widths[j] != 2) return false;
    if (widths[j] == 1) {
      m |= 1 << j;
      ++n1;
    }
  }
  *mask1 = m;
  *mode = n1 == 0 ? 2 : (n1 == S ? 1 : 3);
  return true;
}
int uniform_mask(int bits, int S) { return bits == 1 ? (1 << S) - 1 : 0; }
}  // namespace

size_t mobi_codes_bytes(int64_t N, int64_t K, int S) { return mobi_codes_bytes_bits(N, K, S, 2); }

size_t mobi_codes_bytes_bits(int64_t N, int64_t K, int S, int bits) {
  if (N < 0 || K < 0 || K % 32 != 0 || S < 1 || S > kMaxSlices || bits < 1 || bits > 2) return 0;
  return (size_t)S * (size_t)N * (size_t)(K / 32 * bits) * 4;
}

size_t mobi_codes_bytes_slices(int64_t N, int64_t K, int S, const int* widths) {
  int mode = 0, mask1 = 0;
  if (N < 0 || K < 0 || K % 32 != 0 || !width_mode(S, widths, &mode, &mask1)) return 0;
  size_t words = 0;
  for (int j = 0; j < S; ++j) words += (size_t)N * (size_t)(K / 32 * widths[j]);
  return words * 4;
}

size_t mobi_sz_bytes(int64_t N, int64_t K, int S, int G) {
  if (N < 0 || K < 0 || G <= 0 || K % G != 0 || S < 1 || S > kMaxSlices) return 0;
  return (size_t)S * (size_t)N * (size_t)(K / G) * 4;
}

size_t mobi_route_workspace_bytes(int64_t T, int64_t K, int S) {
  if (T < 0 || K < 0 || S < 1 || S > kMaxSlices) return 0;
  return route_ws_bytes(T, K, S);
}

size_t mobi_gemm_workspace_bytes(int64_t T, int64_t N, int64_t K, int S) {
  if (T < 0 || N < 0 || K < 0 || S < 1 || S > kMaxSlices) return 0;
  size_t b = decode_ws_bytes(N, K);
  const size_t p = prefill_ws_bytes(T, N, K);  // either kernel may be chosen (mobi_gemm_path)
  if (p > b) b = p;
  return align256(b);
}

mobi_status mobi_pack(const void* W, int64_t N, int64_t K, int G, int S, uint32_t* codes, uint32_t* sz,
                      void* stream) {
  g_last_error[0] = 0;
  mobi_status st = check_matrix(N, K, G, S);
  if (st != MOBI_OK) return st;
  if (N == 0 || K == 0) return MOBI_OK;
  if (!W || !codes || !sz) return MOBI_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(sz)) return MOBI_ERR_MISALIGNED;
  return cuda_status(launch_pack(W, N, K, S, codes, sz, static_cast<cudaStream_t>(stream), num_sms(), 0, 128));
}

mobi_status mobi_pack_bits(const void* W, int64_t N, int64_t K, int G, int S, int bits, uint32_t* codes,
                           uint32_t* sz, void* stream) {
  g_last_error[0] = 0;
  if (bits < 1 || bits > 2) return MOBI_ERR_INVALID_ARG;
  if (G != 128 && G != 256 && G != 512) return MOBI_ERR_UNSUPPORTED_SHAPE;
  mobi_status st = check_matrix(N, K, 128, S);
  if (st != MOBI_OK) return st;
  if (K % G != 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return MOBI_OK;
  if (!W || !codes || !sz) return MOBI_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(sz)) return MOBI_ERR_MISALIGNED;
  return cuda_status(
      launch_pack(W, N, K, S, codes, sz, static_cast<cudaStream_t>(stream), num_sms(), uniform_mask(bits, S), G));
}

mobi_status mobi_pack_slices(const void* W, int64_t N, int64_t K, int G, int S, const int* widths, uint32_t* codes,
                             uint32_t* sz, void* stream) {
  g_last_error[0] = 0;
  int mode = 0, mask1 = 0;
  if (!width_mode(S, widths, &mode, &mask1)) return MOBI_ERR_INVALID_ARG;
  if (G != 128 && G != 256 && G != 512) return MOBI_ERR_UNSUPPORTED_SHAPE;
  mobi_status st = check_matrix(N, K, 128, S);
  if (st != MOBI_OK) return st;
  if (K % G != 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (N == 0 || K == 0) return MOBI_OK;
  if (!W || !codes || !sz) return MOBI_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(codes) || !aligned16(sz)) return MOBI_ERR_MISALIGNED;
  return cuda_status(launch_pack(W, N, K, S, codes, sz, static_cast<cudaStream_t>(stream), num_sms(), mask1, G));
}

mobi_status mobi_route(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias, int S,
                       int32_t* k_t, int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  if (T < 0 || K < 0 || S < 1 || S > kMaxSlices) return MOBI_ERR_INVALID_ARG;
  if (K % 128 != 0 || K > kMaxDim || T > kMaxDim) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (!offsets || (T > 0 && (!X || !Wr || !k_t || !perm))) return MOBI_ERR_INVALID_ARG;
  if (T > 0 && K == 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if ((X && !aligned16(X)) || (Wr && !aligned16(Wr)) || (bias && !aligned4(bias)) || (k_t && !aligned4(k_t)) ||
      (perm && !aligned4(perm)) || !aligned4(offsets))
    return MOBI_ERR_MISALIGNED;
  const size_t need = route_ws_bytes(T, K, S);
  if (need > 0 && (!ws || ws_bytes < need)) return MOBI_ERR_WORKSPACE;
  if (ws && !aligned16(ws)) return MOBI_ERR_MISALIGNED;
  return cuda_status(
      launch_route(X, T, K, Wr, bias, S, k_t, perm, offsets, ws, static_cast<cudaStream_t>(stream)));
}

size_t mobi_route_mlp_workspace_bytes(int64_t T, int64_t K, int64_t H) {
  if (T < 0 || K < 0 || H < 1) return 0;
  return route_mlp_ws_bytes(T, K, H, num_sms());
}

mobi_status mobi_route_mlp(const void* X, int64_t T, int64_t K, const float* W1, const float* b1, int64_t H,
                           const float* W2, const float* b2, int S, double tau, double delta, int32_t* k_t,
                           int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  if (T < 0 || K < 0 || H < 1 || S < 1 || S > kMaxSlices) return MOBI_ERR_INVALID_ARG;
  if (!(tau > 0.0) || !std::isfinite(tau) || !(delta > 0.0 && delta < 1.0)) return MOBI_ERR_INVALID_ARG;
  if (K % 128 != 0 || K > kMaxDim || T > kMaxDim || H > kMaxMlpHidden) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (!offsets || (T > 0 && (!X || !k_t || !perm))) return MOBI_ERR_INVALID_ARG;
  if (T > 0 && S > 1 && (!W1 || !W2)) return MOBI_ERR_INVALID_ARG;
  if (T > 0 && K == 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if ((X && !aligned16(X)) || (W1 && !aligned4(W1)) || (b1 && !aligned4(b1)) || (W2 && !aligned4(W2)) ||
      (b2 && !aligned4(b2)) || (k_t && !aligned4(k_t)) || (perm && !aligned4(perm)) || !aligned4(offsets) ||
      (ws && !aligned16(ws)))
    return MOBI_ERR_MISALIGNED;
  const int sms = num_sms();
  const size_t need = S > 1 ? route_mlp_ws_bytes(T, K, H, sms) : 0;
  if (need > 0 && (!ws || ws_bytes < need)) return MOBI_ERR_WORKSPACE;
  // sigmoid(s / tau) > delta  <=>  s > tau * log(delta / (1 - delta))  (the sigmoid is increasing)
  const double thr = tau * std::log(delta / (1.0 - delta));
  return cuda_status(launch_route_mlp(X, T, K, W1, b1, H, W2, b2, S, thr, k_t, perm, offsets, ws,
                                      static_cast<cudaStream_t>(stream), sms));
}

mobi_status mobi_gemm_path(const void* X, int64_t T, int64_t K, const int32_t* k_t, const int32_t* perm,
                           const int32_t* offsets, const uint32_t* codes, const uint32_t* sz, int64_t N, int G,
                           int S, float* Y, void* ws, size_t ws_bytes, void* stream, int path) {
  return mobi_gemm_bits(X, T, K, k_t, perm, offsets, codes, sz, N, G, S, 2, Y, ws, ws_bytes, stream, path);
}

static mobi_status gemm_impl(const void* X, int64_t T, int64_t K, const int32_t* k_t, const int32_t* perm,
                             const int32_t* offsets, const uint32_t* codes, const uint32_t* sz, int64_t N, int G,
                             int S, int bits, int mask1, float* Y, void* ws, size_t ws_bytes, void* stream,
                             int path) {
  mobi_status st = check_matrix(N, K, G, S);
  if (st != MOBI_OK) return st;
  if (T < 0) return MOBI_ERR_INVALID_ARG;
  if (T > kMaxDim) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (path < MOBI_PATH_AUTO || path > MOBI_PATH_PREFILL) return MOBI_ERR_INVALID_ARG;
  if (T == 0 || N == 0) return MOBI_OK;
  if (K == 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (!X || !k_t || !perm || !offsets || !codes || !sz || !Y || !ws) return MOBI_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(codes) || !aligned16(sz) || !aligned16(Y) || !aligned16(ws) ||
      !aligned4(k_t) || !aligned4(perm) || !aligned4(offsets))
    return MOBI_ERR_MISALIGNED;
  const bool decode = path == MOBI_PATH_DECODE || (path == MOBI_PATH_AUTO && T <= 16);
  if (decode && T > 16) return MOBI_ERR_UNSUPPORTED_SHAPE;
  const size_t need = decode ? decode_ws_bytes(N, K) : prefill_ws_bytes(T, N, K);
  if (ws_bytes < need) return MOBI_ERR_WORKSPACE;
  cudaError_t e;
  DeviceStatus* dst = device_status(&e);
  if (!dst) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (decode)
    return cuda_status(launch_decode(X, (int)T, K, k_t, codes, sz, N, S, Y, ws, s, dst, bits, mask1));
  return cuda_status(launch_prefill(X, T, K, k_t, perm, offsets, codes, sz, N, S, Y, ws, s, dst, bits, mask1));
}

mobi_status mobi_gemm_bits(const void* X, int64_t T, int64_t K, const int32_t* k_t, const int32_t* perm,
                           const int32_t* offsets, const uint32_t* codes, const uint32_t* sz, int64_t N, int G,
                           int S, int bits, float* Y, void* ws, size_t ws_bytes, void* stream, int path) {
  g_last_error[0] = 0;
  if (bits < 1 || bits > 2) return MOBI_ERR_INVALID_ARG;
  return gemm_impl(X, T, K, k_t, perm, offsets, codes, sz, N, G, S, bits, uniform_mask(bits, S), Y, ws, ws_bytes,
                   stream, path);
}

mobi_status mobi_gemm_slices(const void* X, int64_t T, int64_t K, const int32_t* k_t, const int32_t* perm,
                             const int32_t* offsets, const uint32_t* codes, const uint32_t* sz, int64_t N, int G,
                             int S, const int* widths, float* Y, void* ws, size_t ws_bytes, void* stream,
                             int path) {
  g_last_error[0] = 0;
  int mode = 0, mask1 = 0;
  if (!width_mode(S, widths, &mode, &mask1)) return MOBI_ERR_INVALID_ARG;
  return gemm_impl(X, T, K, k_t, perm, offsets, codes, sz, N, G, S, mode, mask1, Y, ws, ws_bytes, stream, path);
}

size_t mobi_linear_workspace_bytes(int64_t T, int64_t N, int64_t K, int S) {
  if (T < 0 || N < 0 || K < 0 || S < 1 || S > kMaxSlices) return 0;
  return align256(route_ws_bytes(T, K, S)) + mobi_gemm_workspace_bytes(T, N, K, S);
}

mobi_status mobi_linear(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                        const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S, int32_t* k_t,
                        int32_t* perm, int32_t* offsets, float* Y, void* ws, size_t ws_bytes, void* stream) {
  return mobi_linear_bits(X, T, K, Wr, bias, codes, sz, N, G, S, 2, k_t, perm, offsets, Y, ws, ws_bytes, stream);
}

static mobi_status linear_impl(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                               const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S, int bits,
                               int mask1, int32_t* k_t, int32_t* perm, int32_t* offsets, float* Y, void* ws,
                               size_t ws_bytes, void* stream) {
  mobi_status st = check_matrix(N, K, G, S);
  if (st != MOBI_OK) return st;
  if (T < 0) return MOBI_ERR_INVALID_ARG;
  if (T > kMaxDim) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (!offsets || (T > 0 && (!X || !Wr || !k_t || !perm))) return MOBI_ERR_INVALID_ARG;
  if (T > 0 && K == 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (T > 0 && N > 0 && (!codes || !sz || !Y || !ws)) return MOBI_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (Wr && !aligned16(Wr)) || (bias && !aligned4(bias)) || (k_t && !aligned4(k_t)) ||
      (perm && !aligned4(perm)) || !aligned4(offsets) || (codes && !aligned16(codes)) || (sz && !aligned16(sz)) ||
      (Y && !aligned16(Y)) || (ws && !aligned16(ws)))
    return MOBI_ERR_MISALIGNED;
  const size_t route_ws = align256(route_ws_bytes(T, K, S));
  const bool decode = T <= 16;
  const size_t need = route_ws + (T > 0 && N > 0 ? (decode ? decode_ws_bytes(N, K) : prefill_ws_bytes(T, N, K)) : 0);
  if (need > 0 && (!ws || ws_bytes < need)) return MOBI_ERR_WORKSPACE;
  cudaError_t e;
  DeviceStatus* dst = device_status(&e);
  if (!dst) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  e = launch_route(X, T, K, Wr, bias, S, k_t, perm, offsets, ws, s);
  if (e != cudaSuccess || T == 0 || N == 0) return cuda_status(e);
  void* gws = static_cast<uint8_t*>(ws) + route_ws;
  // For up to 16 tokens the decode kernel is a programmatic dependent of the
  // routing kernel just launched: its launch and set-up overlap the routing.
  if (decode)
    return cuda_status(launch_decode(X, (int)T, K, k_t, codes, sz, N, S, Y, gws, s, dst, bits, mask1));
  return cuda_status(launch_prefill(X, T, K, k_t, perm, offsets, codes, sz, N, S, Y, gws, s, dst, bits, mask1));
}

mobi_status mobi_linear_bits(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                             const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S, int bits,
                             int32_t* k_t, int32_t* perm, int32_t* offsets, float* Y, void* ws, size_t ws_bytes,
                             void* stream) {
  g_last_error[0] = 0;
  if (bits < 1 || bits > 2) return MOBI_ERR_INVALID_ARG;
  return linear_impl(X, T, K, Wr, bias, codes, sz, N, G, S, bits, uniform_mask(bits, S), k_t, perm, offsets, Y, ws,
                     ws_bytes, stream);
}

mobi_status mobi_linear_slices(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                               const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S, const int* widths,
                               int32_t* k_t, int32_t* perm, int32_t* offsets, float* Y, void* ws, size_t ws_bytes,
                               void* stream) {
  g_last_error[0] = 0;
  int mode = 0, mask1 = 0;
  if (!width_mode(S, widths, &mode, &mask1)) return MOBI_ERR_INVALID_ARG;
  return linear_impl(X, T, K, Wr, bias, codes, sz, N, G, S, mode, mask1, k_t, perm, offsets, Y, ws, ws_bytes,
                     stream);
}

static_assert(MOBI_MAX_GROUP == kMaxGroup, "group size of the header and the kernels");

static mobi_status check_grouped(const mobi_linear_problem* problems, int count, int G, int S, size_t* need) {
  *need = 0;
  if (!problems || count < 1 || count > MOBI_MAX_GROUP) return MOBI_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const mobi_linear_problem& p = problems[i];
    mobi_status st = check_matrix(p.N, p.K, G, S);
    if (st != MOBI_OK) return st;
    if (p.T < 0) return MOBI_ERR_INVALID_ARG;
    if (p.T > 16) return MOBI_ERR_UNSUPPORTED_SHAPE;
    if (!p.offsets || (p.T > 0 && (!p.X || !p.Wr || !p.k_t || !p.perm))) return MOBI_ERR_INVALID_ARG;
    if (p.T > 0 && p.K == 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
    if (p.T > 0 && p.N > 0 && (!p.codes || !p.sz || !p.Y)) return MOBI_ERR_INVALID_ARG;
    if ((p.X && !aligned16(p.X)) || (p.Wr && !aligned16(p.Wr)) || (p.bias && !aligned4(p.bias)) ||
        (p.k_t && !aligned4(p.k_t)) || (p.perm && !aligned4(p.perm)) || !aligned4(p.offsets) ||
        (p.codes && !aligned16(p.codes)) || (p.sz && !aligned16(p.sz)) || (p.Y && !aligned16(p.Y)))
      return MOBI_ERR_MISALIGNED;
    if (p.T > 0 && p.N > 0) *need += align256(decode_ws_bytes(p.N, p.K));
  }
  return MOBI_OK;
}

size_t mobi_linear_grouped_workspace_bytes(const mobi_linear_problem* problems, int count, int S) {
  size_t need = 0;
  if (check_grouped(problems, count, 128, S, &need) != MOBI_OK) return 0;
  return need;
}

mobi_status mobi_linear_grouped(const mobi_linear_problem* problems, int count, int G, int S, void* ws,
                                size_t ws_bytes, void* stream) {
  return mobi_linear_grouped_bits(problems, count, G, S, 2, ws, ws_bytes, stream);
}

static mobi_status linear_grouped_impl(const mobi_linear_problem* problems, int count, int G, int S, int bits,
                                       int mask1, void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  mobi_status st = check_grouped(problems, count, G, S, &need);
  if (st != MOBI_OK) return st;
  if (ws && !aligned16(ws)) return MOBI_ERR_MISALIGNED;
  if (need > 0 && (!ws || ws_bytes < need)) return MOBI_ERR_WORKSPACE;
  cudaError_t e;
  DeviceStatus* dst = device_status(&e);
  if (!dst) return cuda_status(e);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  RouteSmallGroup rg = {};
  rg.G = count;
  DecodeJob jobs[MOBI_MAX_GROUP];
  uint8_t* w = static_cast<uint8_t*>(ws);
  for (int i = 0; i < count; ++i) {
    const mobi_linear_problem& p = problems[i];
    rg.p[i] = RouteSmallProblem{static_cast<const __nv_bfloat16*>(p.X), p.Wr, p.bias, p.k_t, p.perm, p.offsets, p.K,
                                (int)p.T};
    jobs[i] = DecodeJob{p.X, p.k_t, p.codes, p.sz, p.Y, nullptr, p.N, p.K, (int)p.T, bits, mask1};
    if (p.T > 0 && p.N > 0) {
      jobs[i].partial = reinterpret_cast<float*>(w);
      w += align256(decode_ws_bytes(p.N, p.K));
    }
  }
  e = launch_route_small_grouped(rg, S, s);
  if (e != cudaSuccess) return cuda_status(e);
  // As in mobi_linear: the decode launches are programmatic dependents of the
  // routing launch.
  return cuda_status(launch_decode_grouped(jobs, count, S, s, dst));
}

mobi_status mobi_linear_grouped_bits(const mobi_linear_problem* problems, int count, int G, int S, int bits,
                                     void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  if (bits < 1 || bits > 2) return MOBI_ERR_INVALID_ARG;
  return linear_grouped_impl(problems, count, G, S, bits, uniform_mask(bits, S), ws, ws_bytes, stream);
}

mobi_status mobi_linear_grouped_slices(const mobi_linear_problem* problems, int count, int G, int S,
                                       const int* widths, void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  int mode = 0, mask1 = 0;
  if (!width_mode(S, widths, &mode, &mask1)) return MOBI_ERR_INVALID_ARG;
  return linear_grouped_impl(problems, count, G, S, mode, mask1, ws, ws_bytes, stream);
}

static mobi_status check_gemm_grouped(const mobi_gemm_problem* problems, int count, int G, int S, size_t* need) {
  *need = 0;
  if (!problems || count < 1 || count > MOBI_MAX_GROUP) return MOBI_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const mobi_gemm_problem& p = problems[i];
    mobi_status st = check_matrix(p.N, p.K, G, S);
    if (st != MOBI_OK) return st;
    if (p.T < 0) return MOBI_ERR_INVALID_ARG;
    if (p.T > 16) return MOBI_ERR_UNSUPPORTED_SHAPE;
    if (p.T == 0 || p.N == 0) continue;
    if (p.K == 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
    if (!p.X || !p.k_t || !p.codes || !p.sz || !p.Y) return MOBI_ERR_INVALID_ARG;
    if (!aligned16(p.X) || !aligned16(p.codes) || !aligned16(p.sz) || !aligned16(p.Y) || !aligned4(p.k_t))
      return MOBI_ERR_MISALIGNED;
    *need += align256(decode_ws_bytes(p.N, p.K));
  }
  return MOBI_OK;
}

size_t mobi_gemm_grouped_workspace_bytes(const mobi_gemm_problem* problems, int count, int S) {
  size_t need = 0;
  if (check_gemm_grouped(problems, count, 128, S, &need) != MOBI_OK) return 0;
  return need;
}

mobi_status mobi_gemm_grouped(const mobi_gemm_problem* problems, int count, int G, int S, void* ws,
                              size_t ws_bytes, void* stream) {
  return mobi_gemm_grouped_bits(problems, count, G, S, 2, ws, ws_bytes, stream);
}

static mobi_status gemm_grouped_impl(const mobi_gemm_problem* problems, int count, int G, int S, int bits,
                                     int mask1, void* ws, size_t ws_bytes, void* stream) {
  size_t need = 0;
  mobi_status st = check_gemm_grouped(problems, count, G, S, &need);
  if (st != MOBI_OK) return st;
  if (ws && !aligned16(ws)) return MOBI_ERR_MISALIGNED;
  if (need > 0 && (!ws || ws_bytes < need)) return MOBI_ERR_WORKSPACE;
  cudaError_t e;
  DeviceStatus* dst = device_status(&e);
  if (!dst) return cuda_status(e);
  DecodeJob jobs[MOBI_MAX_GROUP];
  uint8_t* w = static_cast<uint8_t*>(ws);
  for (int i = 0; i < count; ++i) {
    const mobi_gemm_problem& p = problems[i];
    jobs[i] = DecodeJob{p.X, p.k_t, p.codes, p.sz, p.Y, nullptr, p.N, p.K, (int)p.T, bits, mask1};
    if (p.T > 0 && p.N > 0) {
      jobs[i].partial = reinterpret_cast<float*>(w);
      w += align256(decode_ws_bytes(p.N, p.K));
    }
  }
  return cuda_status(launch_decode_grouped(jobs, count, S, static_cast<cudaStream_t>(stream), dst));
}

mobi_status mobi_gemm_grouped_bits(const mobi_gemm_problem* problems, int count, int G, int S, int bits, void* ws,
                                   size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  if (bits < 1 || bits > 2) return MOBI_ERR_INVALID_ARG;
  return gemm_grouped_impl(problems, count, G, S, bits, uniform_mask(bits, S), ws, ws_bytes, stream);
}

mobi_status mobi_gemm_grouped_slices(const mobi_gemm_problem* problems, int count, int G, int S, const int* widths,
                                     void* ws, size_t ws_bytes, void* stream) {
  g_last_error[0] = 0;
  int mode = 0, mask1 = 0;
  if (!width_mode(S, widths, &mode, &mask1)) return MOBI_ERR_INVALID_ARG;
  return gemm_grouped_impl(problems, count, G, S, mode, mask1, ws, ws_bytes, stream);
}

mobi_status mobi_gemm(const void* X, int64_t T, int64_t K, const int32_t* k_t, const int32_t* perm,
                      const int32_t* offsets, const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S,
                      float* Y, void* ws, size_t ws_bytes, void* stream) {
  return mobi_gemm_path(X, T, K, k_t, perm, offsets, codes, sz, N, G, S, Y, ws, ws_bytes, stream,
                        MOBI_PATH_AUTO);
}

mobi_status mobi_sync_check(void* stream) {
  g_last_error[0] = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_status(e);
  DeviceStatus* dst = device_status(&e);
  if (!dst) return cuda_status(e);
  DeviceStatus h;
  e = cudaMemcpy(&h, dst, sizeof h, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_status(e);
  if (h.error == 0) return MOBI_OK;
  const DeviceStatus zero = {};
  e = cudaMemcpy(dst, &zero, sizeof zero, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_status(e);
  if (h.error & kErrTimeout) {
    snprintf(g_last_error, sizeof g_last_error, "a bounded wait ran out in a kernel (wait site 0x%x)", h.where);
    return MOBI_ERR_TIMEOUT;
  }
  note_message("an activation of a decode call (T <= 16) had |x| >= 2^31");
  return MOBI_ERR_INVALID_ARG;  // kErrInputRange
}

mobi_status mobi_debug_set_wait_limit(int64_t limit) {
  if (limit < 0) return MOBI_ERR_INVALID_ARG;
  const int d = current_device();
  if (d < 0) return MOBI_ERR_CUDA;
  g_wait_limit[d].store((uint64_t)limit);
  return MOBI_OK;
}

}  // extern "C"
