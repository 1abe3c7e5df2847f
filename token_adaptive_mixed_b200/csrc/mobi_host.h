// mobi_host.h — host-side helpers shared by the libmobi launchers: per-device
// status word, SM count, tensor-map encoding through the driver entry point.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "mobi_device.cuh"

namespace mobi {

// Device address of the per-device DeviceStatus (set up on first use per device).
DeviceStatus* device_status(cudaError_t* err);
// Wait limit for bounded device waits on the current device.
uint64_t wait_limit();
// Record a failure description for mobi_last_error (thread-local) and return e.
cudaError_t note_error(const char* where, cudaError_t e);
// Multiprocessor count of the current device (cached).
int num_sms();
// Opt a kernel into `bytes` of dynamic shared memory (idempotent).
cudaError_t set_smem(const void* func, int bytes);

// 2-D tiled tensor map over a row-major [rows][cols] array of `elem_bytes`
// elements (cols innermost), box [box_rows][box_cols]; swizzle_bytes is 0 (none),
// 32, 64 or 128 (the shared-memory swizzle span of the copied tile).
bool make_tmap_2d(CUtensorMap* map, const void* base, int elem_bytes, uint64_t cols, uint64_t rows,
                  uint64_t row_stride_bytes, uint32_t box_cols, uint32_t box_rows, int swizzle_bytes);

}  // namespace mobi
