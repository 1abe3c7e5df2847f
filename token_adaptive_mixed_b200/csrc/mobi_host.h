// mobi_host.h — host-side helpers shared by the libmobi launchers: per-device
// status word, SM count, tensor-map encoding through the driver entry point.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cuda_bf16.h>

#include <cstdint>

#include "../../include/mobi.h"
#include "mobi_device.cuh"

namespace mobi {

// Device address of the per-device DeviceStatus (set up on first use per device).
DeviceStatus* device_status(cudaError_t* err);
// Wait limit for bounded device waits on the current device.
uint64_t wait_limit();
// Record a failure description for mobi_last_error (thread-local) and return e.
cudaError_t note_error(const char* where, cudaError_t e);
// Record a plain message for mobi_last_error.
void note_message(const char* msg);
// Clear the message mobi_last_error returns (each entry point starts with this).
void clear_message();
// C-ABI status of a CUDA error: MOBI_OK, or MOBI_ERR_CUDA with the error kept
// for mobi_last_error and a sticky launch error cleared.
mobi_status status_of(cudaError_t e);
// Multiprocessor count of the current device (cached).
int num_sms();
// Opt a kernel into `bytes` of dynamic shared memory (idempotent).
cudaError_t set_smem(const void* func, int bytes);

// 2-D tiled tensor map over a row-major [rows][cols] array of `elem_bytes`
// elements (cols innermost), box [box_rows][box_cols]; swizzle_bytes is 0 (none),
// 32, 64 or 128 (the shared-memory swizzle span of the copied tile).
bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes);

// ---- groups of independent small problems (one launch each step) -------------------
//
// Problem tables travel as __grid_constant__ kernel parameters, so a CUDA graph
// captures them by value and no device memory holds them.
constexpr int kMaxGroup = 16;
// Slices per packed layer: up to four (e.g. four 1-bit slices for 1..4 bits).
constexpr int kMaxSlices = 4;

struct RouteSmallProblem {
  const __nv_bfloat16* X;
  const float* Wr;
  const float* bias;
  int32_t* k_t;
  int32_t* perm;
  int32_t* offsets;
  int64_t K;
  int T;
};
template <int MG>
struct RouteSmallGroupT {
  RouteSmallProblem p[MG];
  int G;
};
using RouteSmallGroup = RouteSmallGroupT<kMaxGroup>;
cudaError_t launch_route_small_grouped(const RouteSmallGroup& grp, int S, cudaStream_t stream);

// One decode problem (T <= 16): inputs, k_t, and the output Y.
struct DecodeJob {
  const void* X;
  const int32_t* k_t;
  const uint32_t* codes;
  const uint32_t* sz;
  float* Y;
  float* partial;  // scratch of decode_ws_bytes(N, K) bytes
  int64_t N, K;
  int T;
  int bits;   // 2 or 1: every slice that wide (16 or 32 codes per word); 3: widths per slice (mask1)
  int mask1;  // bits == 3: bit s set = slice s has 1-bit codes; the slices are stored one after another
};
// Decode scratch of one problem: the per-chunk partial sums when K spans more
// than one 1024-column chunk.
size_t decode_ws_bytes(int64_t N, int64_t K);
// Y[t][n] = sum over chunks c (in order) of partial[c][t][n] (T N % 4 == 0),
// launched as a programmatic dependent of the kernel before it.
cudaError_t launch_chunk_reduce(const float* partial, float* Y, int64_t T, int64_t N, int nch, cudaStream_t stream);
// Decode GEMMs of up to kMaxGroup problems: one launch per fragment class
// (T <= 8, T <= 16) and code width present, plus one chunk-reduction launch.
cudaError_t launch_decode_grouped(const DecodeJob* jobs, int G, int S, cudaStream_t stream, DeviceStatus* st);

}  // namespace mobi
