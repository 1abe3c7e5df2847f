// mobi_pack.cu — MoBiSlice recursive residual quantisation on sm_100a.
//
// MoBiQuant explainer [ja] §2.1 / [en] §2.A: R_1 = W, W_s = Q(R_s),
// R_{s+1} = R_s - W_s, with Q the asymmetric min-max round-to-nearest of each
// G-wide group (the quantiser written out in include/mobi.h): b-bit codes,
// L = 2^b - 1 steps (b = 2 for the method's slices, b = 1 for generic ones,
// one width per slice), G = 128, 256 or 512.
//
// Work split: one warp per (row n, chunk of 512 columns); lane l owns the 16
// consecutive weights k = 512c + 16l .. +15, i.e. exactly one 2-bit-field
// word per slice. The G/16 lanes of a group reduce min/max with xor shuffles.
// 2-bit codes leave as 128-bit stores (4 lanes' words gathered into one lane),
// so each slice's 128 bytes per warp are one coalesced transaction. 1-bit
// codes are stored at 1 bit per weight: lanes 2m and 2m + 1 merge their words
// (the odd lane's codes on the odd bits) into one 32-code word, and four such
// words leave as one 128-bit store (64 bytes per warp and slice). Scale/zero
// words are written per 128-column sub-group, so a wider group's word appears
// once per sub-group (the layout the GEMM kernels read).
//
// Bit-exactness: IEEE division (__fdiv_rn), round-to-nearest-even (rintf,
// __float2half_rn), explicit _rn multiply/subtract so that nothing is
// contracted, no flush-to-zero (no fast-math).
#include <cstdint>

#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

// Slice s has 1-bit codes when bit s of mask1 is set, 2-bit codes otherwise;
// the slices are stored one after another, each in the layout of its width.
__global__ void __launch_bounds__(256) pack_kernel(const __half* __restrict__ W, int64_t N, int64_t K,
                                                   int S, int mask1, int glanes, uint32_t* __restrict__ codes,
                                                   uint32_t* __restrict__ sz) {
  const int lane = threadIdx.x & 31;
  const int64_t ngroups = K / 128;
  const int64_t nchunks = (ngroups + 3) / 4;
  const int64_t nwords = K / 16;
  const int64_t units = N * nchunks;
  const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x / 32);
  int64_t unit = (int64_t)blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);

  for (; unit < units; unit += warps_total) {
    const int64_t n = unit / nchunks;
    const int64_t c = unit % nchunks;
    const int64_t g = 4 * c + (lane >> 3);  // this lane's group
    const bool valid = g < ngroups;
    const int64_t k0 = 512 * c + 16 * lane;

    float R[16];
    if (valid) {
      const uint4* src = reinterpret_cast<const uint4*>(W + n * K + k0);
      uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
      const uint32_t u[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        __half2 h = *reinterpret_cast<const __half2*>(&u[i]);
        R[2 * i] = __low2float(h);
        R[2 * i + 1] = __high2float(h);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) R[i] = 0.0f;
    }

    int64_t slice_base = 0;  // word offset of slice s
    for (int s = 0; s < S; ++s) {
      const int bits = ((mask1 >> s) & 1) ? 1 : 2;
      const float L = (float)((1 << bits) - 1);  // steps between min and max
      float mn = R[0], mx = R[0];
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        mn = fminf(mn, R[i]);
        mx = fmaxf(mx, R[i]);
      }
      for (int o = 1; o < glanes; o <<= 1) {  // the G / 16 lanes of this group
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      }
      float sc = __fdiv_rn(__fsub_rn(mx, mn), L);
      sc = fmaxf(sc, 0x1p-14f);
      const __half scale_h = __float2half_rn(sc);
      const float step = __half2float(scale_h);
      float zf = rintf(__fdiv_rn(-mn, step));
      zf = fminf(fmaxf(zf, 0.0f), L);
      const int z = (int)zf;

      uint32_t word = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float qf = rintf(__fdiv_rn(R[i], step)) + (float)z;
        qf = fminf(fmaxf(qf, 0.0f), L);
        const int q = (int)qf;
        word |= (uint32_t)q << (2 * i);
        R[i] = __fsub_rn(R[i], __fmul_rn((float)(q - z), step));
      }

      if (bits == 1) {
        // 32 codes per word: this lane's 16 on the even bits, the next lane's on
        // the odd bits (valid in even lanes); lanes 8j, 8j + 2, 8j + 4, 8j + 6
        // hold one group's four words, gathered into lane 8j: one uint4.
        const uint32_t dense = word | (__shfl_down_sync(0xffffffffu, word, 1) << 1);
        const uint32_t d1 = __shfl_down_sync(0xffffffffu, dense, 2);
        const uint32_t d2 = __shfl_down_sync(0xffffffffu, dense, 4);
        const uint32_t d3 = __shfl_down_sync(0xffffffffu, dense, 6);
        if (valid && (lane & 7) == 0) {
          uint4* dst = reinterpret_cast<uint4*>(codes + slice_base + n * (K / 32) + 16 * c + (lane >> 1));
          *dst = make_uint4(dense, d1, d2, d3);
        }
      } else {
        // Gather 4 consecutive lanes' words into the first of them: one uint4.
        const uint32_t w1 = __shfl_down_sync(0xffffffffu, word, 1);
        const uint32_t w2 = __shfl_down_sync(0xffffffffu, word, 2);
        const uint32_t w3 = __shfl_down_sync(0xffffffffu, word, 3);
        if (valid && (lane & 3) == 0) {
          uint4* dst = reinterpret_cast<uint4*>(codes + slice_base + n * nwords + 32 * c + lane);
          *dst = make_uint4(word, w1, w2, w3);
        }
      }
      if (valid && (lane & 7) == 0) {
        const uint32_t zbits = (uint32_t)__half_as_ushort(__int2half_rn(z));
        sz[((int64_t)s * ngroups + g) * N + n] = (uint32_t)__half_as_ushort(scale_h) | (zbits << 16);
      }
      slice_base += N * (K / 32) * bits;
    }
  }
}

cudaError_t launch_pack(const void* W, int64_t N, int64_t K, int S, uint32_t* codes, uint32_t* sz,
                        cudaStream_t stream, int num_sms, int mask1, int G) {
  const int64_t nchunks = (K / 128 + 3) / 4;
  const int64_t units = N * nchunks;
  const int warps_per_block = 8;
  int64_t blocks = (units + warps_per_block - 1) / warps_per_block;
  const int64_t cap = (int64_t)num_sms * 16;  // grid-stride beyond ~16 blocks per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  pack_kernel<<<(unsigned)blocks, 32 * warps_per_block, 0, stream>>>(
      static_cast<const __half*>(W), N, K, S, mask1, G / 16, codes, sz);
  return note_error("kernel launch", cudaGetLastError());
}

}  // namespace mobi
