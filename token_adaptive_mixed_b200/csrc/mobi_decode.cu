// mobi_decode.cu — decode GEMM (T <= 16 tokens) of the token-routed mixed-bit
// linear layer on sm_100a.
//
// y[t,n] = sum_{s < k_t} sum_g scale[s,g,n] * sum_{k in g} x[t,k] (q[s,n,k] - z[s,g,n])
// (MoBiQuant explainer [ja] §2.1 W^(b) = sum W_e; [en] §2.A "Elasticity").
// Only the slices up to the batch's largest k_t are read ([en] §3: fetch only
// the slices that are needed).
//
// Exact operands on the tensor cores. A 2-bit code q sitting at bit 2f of a
// byte is, read as a bf16 bit pattern, the subnormal value q * 4^f * 2^-133
// (bf16 values with exponent field 0 or 1 are linear in their bit pattern).
// So `word & (0x00030003 << 2f)` (after an optional 8-bit shift) is a pair of
// exact A-operand values, one AND per two weights. The activations are staged
// once per call as x * 2^96 / 4^f (exact in bf16 for |x| < 2^31), so every
// product is q * x * 2^-37 exactly and every field carries the same weight.
// The zero point is folded in once per (row, group): sum_k x (q - z) =
// sum_k x q - z * sum_k x, with sum_k x prepared in fp64 and rounded once.
// fp32 accumulation happens in the tensor core (mma.sync m16n8k16) and in the
// per-group promotion y += scale * 2^37 * acc - scale * z * xsum.
//
// Work split: CTA = 64 rows x 8 groups (1024 columns), 4 warps; warp w handles
// groups 2w, 2w+1 for all four 16-row tiles, so each activation fragment is
// read from shared memory once and used for 4 tiles x k slices. Codes, scales
// and the staged activations arrive by TMA, one mbarrier per slice, so slice 0
// is computed while slices 1..k-1 are still in flight. Column splits are
// combined deterministically: every CTA writes its partial to the workspace
// and the last CTA of a row block (atomic ticket) sums them in order.
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/mobi.h"
#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

constexpr int kDecRows = 64;      // rows per CTA
constexpr int kDecGroups = 8;     // 128-wide groups per CTA
constexpr int kDecThreads = 256;  // 8 warps, one 128-wide group each
constexpr float kTwo96 = 79228162514264337593543950336.0f;  // 2^96
constexpr float kTwo37 = 137438953472.0f;                   // 2^37

// ---- staging of the activations ------------------------------------------------
//
// Xd[g][j][lane][nb][2] (uint32 = bf16 pair) is the B fragment of k16 step j
// (j = 4h + f) of group g for lane (gid = lane/4, t4 = lane%4) and token
// gid + 8nb. Register ih in {0,1} holds the pair e in {0,1} at physical column
//   k = 128g + 32 t4 + 16 ih + 4h + f + 8e,
// scaled by 2^(96 - 2f). xs[g][t] = sum of x[t, group g] (fp64, stored fp32).
// meta[0] = max k_t; meta[1..] are the per-row-block tickets (zeroed here).
__global__ void __launch_bounds__(256) decode_prep_kernel(const __nv_bfloat16* __restrict__ X, int T,
                                                          int64_t K, int NB, const int32_t* __restrict__ k_t,
                                                          uint32_t* __restrict__ Xd, float* __restrict__ xs,
                                                          int32_t* __restrict__ meta, int64_t n_tickets,
                                                          DeviceStatus* st) {
  const int64_t g = blockIdx.x;
  const int tid = threadIdx.x;
  // The decode kernel may start now: it only reads these outputs after its
  // grid-dependency wait.
  asm volatile("griddepcontrol.launch_dependents;");
  {
    const int j = tid >> 5, lane = tid & 31;
    const int gid = lane >> 2, t4 = lane & 3, h = j >> 2, f = j & 3;
    const float mult = kTwo96 / (float)(1 << (2 * f));
    bool bad = false;
    for (int nb = 0; nb < NB; ++nb) {
      const int tok = gid + 8 * nb;
      uint32_t reg[2];
#pragma unroll
      for (int ih = 0; ih < 2; ++ih) {
        uint32_t pair = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int64_t k = 128 * g + 32 * t4 + 16 * ih + 4 * h + f + 8 * e;
          float x = 0.0f;
          if (tok < T) x = __bfloat162float(X[(int64_t)tok * K + k]);
          bad |= !(fabsf(x) < 0x1p31f);
          const __nv_bfloat16 b = __float2bfloat16_rn(x * mult);  // exact: power-of-two scaling
          pair |= (uint32_t)__bfloat16_as_ushort(b) << (16 * e);
        }
        reg[ih] = pair;
      }
      uint32_t* dst = Xd + (((g * 8 + j) * 32 + lane) * NB + nb) * 2;
      dst[0] = reg[0];
      dst[1] = reg[1];
    }
    if (bad) report_error(st, kErrInputRange, 0x100);
  }
  {
    // Group sums: thread (tok = tid/16, part = tid%16) adds 8 columns in fp64,
    // then a fixed xor tree over the 16 parts.
    const int tok = tid >> 4, part = tid & 15;
    double s = 0.0;
    if (tok < T) {
      const __nv_bfloat16* p = X + (int64_t)tok * K + 128 * g + 8 * part;
#pragma unroll
      for (int i = 0; i < 8; ++i) s += (double)__bfloat162float(p[i]);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (part == 0) xs[g * 16 + tok] = (float)s;
  }
  if (g == 0 && tid == 0) {
    int km = 1;
    for (int t = 0; t < T; ++t) km = max(km, (int)k_t[t]);
    meta[0] = km;
  }
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + tid; i < n_tickets; i += (int64_t)gridDim.x * blockDim.x)
    meta[1 + i] = 0;
}

// ---- the decode kernel ------------------------------------------------------------

struct DecSmem {
  // Codes of one slice: two TMA boxes of [64 rows][32 words] with 128-byte
  // swizzle (16-byte chunk j of row r sits at chunk j ^ (r & 7)), so the eight
  // rows a warp reads in one instruction fall on different banks.
  uint32_t codes[3][2][kDecRows][32];            // 48 KB, 1024-byte aligned
  uint32_t sz[3][kDecGroups][kDecRows];          // [slice][group][row]          6 KB
  float xs[kDecGroups][16];                      // group sums                 512 B
  int32_t kt[16];
  int32_t kmax;
  int32_t is_last;
  uint64_t bar[3];
};

__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Words 2*t4 and 2*t4+1 of group gi of `row` from the swizzled code tile.
__device__ __forceinline__ uint2 code_pair(const uint32_t (*tile)[kDecRows][32], int row, int gi, int t4) {
  const int half = gi >> 2;
  const int chunk = ((gi & 3) << 1) + (t4 >> 1);
  const int phys = chunk ^ (row & 7);
  return *reinterpret_cast<const uint2*>(&tile[half][row][phys * 4 + ((t4 & 1) << 1)]);
}

constexpr size_t kDecSmemXd = (sizeof(DecSmem) + 127) / 128 * 128;

template <int NB>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(
    const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_sz,
    const uint32_t* __restrict__ Xd, const float* __restrict__ xs_g, const int32_t* __restrict__ k_t,
    int32_t* __restrict__ meta, int T, int64_t N, int64_t ngroups, int S, float* __restrict__ partial,
    float* __restrict__ Y, DeviceStatus* st, uint64_t limit) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  DecSmem& sm = *reinterpret_cast<DecSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* xd_s = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(&sm) + kDecSmemXd);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, t4 = lane & 3;
  const int64_t rb = blockIdx.x;                  // row block
  const int64_t ch = blockIdx.y;                  // column chunk (8 groups)
  const int nch = gridDim.y;
  const int64_t g0 = ch * kDecGroups;
  const int ngc = (int)(ngroups - g0 < kDecGroups ? ngroups - g0 : kDecGroups);

  // k_t was written before this call's staging kernel started, so it can be
  // read before the grid dependency is resolved.
  if (tid < 16) sm.kt[tid] = tid < T ? k_t[tid] : 0;
  if (tid == 0) {
    for (int s = 0; s < 3; ++s) mbar_init(&sm.bar[s], 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (tid == 0) {
    int km = 1;
    for (int t = 0; t < T; ++t) km = max(km, (int)sm.kt[t]);
    km = min(km, S);
    sm.kmax = km;
    const uint32_t xd_bytes = (uint32_t)ngc * 2048u * NB;
    const uint32_t xs_bytes = (uint32_t)ngc * 64u;
    for (int s = 0; s < km; ++s) {
      const uint32_t bytes = sizeof(sm.codes[0]) + sizeof(sm.sz[0]) + (s == 0 ? xd_bytes + xs_bytes : 0u);
      mbar_arrive_expect_tx(&sm.bar[s], bytes);
      const int y = (int)(s * N + rb * kDecRows);
      tma_load_2d(&sm.codes[s][0][0][0], &tm_codes, (int)(g0 * 8), y, &sm.bar[s]);
      tma_load_2d(&sm.codes[s][1][0][0], &tm_codes, (int)(g0 * 8 + 32), y, &sm.bar[s]);
      tma_load_2d(&sm.sz[s][0][0], &tm_sz, (int)(rb * kDecRows), (int)(s * ngroups + g0), &sm.bar[s]);
    }
  }
  // The staged activations, group sums and tickets come from the staging
  // kernel launched just before (programmatic dependent launch).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (tid == 0) {
    bulk_g2s(xd_s, Xd + g0 * 512 * NB, (uint32_t)ngc * 2048u * NB, &sm.bar[0]);
    bulk_g2s(&sm.xs[0][0], xs_g + g0 * 16, (uint32_t)ngc * 64u, &sm.bar[0]);
  }
  __syncthreads();
  const int kmax = sm.kmax;

  // yt[r][2 nb + 0] = row 16r+gid, tokens (2t4, 2t4+1) + 8nb; [2 nb + 1] = row +8.
  float2 yt[4][2 * NB];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int i = 0; i < 2 * NB; ++i) yt[r][i] = make_float2(0.0f, 0.0f);

  const int gi = warp;  // this warp's group within the chunk
  bool ok = true;
  if (gi < ngc || warp == 0) {
    for (int s = 0; s < kmax; ++s) {
      if (!mbar_wait(&sm.bar[s], 0, limit, st, 0x200 + s)) {
        ok = false;
        mbar_wait(&sm.bar[s], 0, kDefaultWaitLimit, st, 0x210 + s);  // drain the copies in flight
        continue;
      }
      if (!ok || gi >= ngc) continue;
      // B fragments of the 8 k16 steps, zeroed for tokens that do not take slice s.
      uint32_t b[8][2 * NB];
      bool on[NB];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) on[nb] = sm.kt[gid + 8 * nb] > s;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const uint32_t* src = xd_s + ((gi * 8 + j) * 32 + lane) * NB * 2;
        if constexpr (NB == 2) {
          const uint4 v = *reinterpret_cast<const uint4*>(src);
          b[j][0] = on[0] ? v.x : 0u; b[j][1] = on[0] ? v.y : 0u;
          b[j][2] = on[1] ? v.z : 0u; b[j][3] = on[1] ? v.w : 0u;
        } else {
          const uint2 v = *reinterpret_cast<const uint2*>(src);
          b[j][0] = on[0] ? v.x : 0u; b[j][1] = on[0] ? v.y : 0u;
        }
      }
      float2 xsv[NB];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const int tk = 2 * t4 + 8 * nb;
        xsv[nb] = make_float2(sm.kt[tk] > s ? sm.xs[gi][tk] : 0.0f, sm.kt[tk + 1] > s ? sm.xs[gi][tk + 1] : 0.0f);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int rowA = 16 * r + gid, rowB = rowA + 8;
        const uint2 wa = code_pair(sm.codes[s], rowA, gi, t4);
        const uint2 wb = code_pair(sm.codes[s], rowB, gi, t4);
        float d[NB][4];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) d[nb][0] = d[nb][1] = d[nb][2] = d[nb][3] = 0.0f;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t a0w = wa.x >> (8 * h), a2w = wa.y >> (8 * h);
          const uint32_t a1w = wb.x >> (8 * h), a3w = wb.y >> (8 * h);
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            const uint32_t m = 0x00030003u << (2 * f);
            const int j = 4 * h + f;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
              mma_bf16_16816(d[nb], a0w & m, a1w & m, a2w & m, a3w & m, b[j][2 * nb], b[j][2 * nb + 1]);
          }
        }
        const uint32_t szA = sm.sz[s][gi][rowA], szB = sm.sz[s][gi][rowB];
        const float scA = __half2float(__ushort_as_half((unsigned short)(szA & 0xffffu)));
        const float zA = __half2float(__ushort_as_half((unsigned short)(szA >> 16)));
        const float scB = __half2float(__ushort_as_half((unsigned short)(szB & 0xffffu)));
        const float zB = __half2float(__ushort_as_half((unsigned short)(szB >> 16)));
        // Packed fp32x2 FMAs: y += scale 2^37 * acc - scale z * xsum (both constants exact).
        const float2 aA = make_float2(scA * kTwo37, scA * kTwo37), cA = make_float2(-scA * zA, -scA * zA);
        const float2 aB = make_float2(scB * kTwo37, scB * kTwo37), cB = make_float2(-scB * zB, -scB * zB);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          yt[r][2 * nb] = __ffma2_rn(cA, xsv[nb], __ffma2_rn(aA, make_float2(d[nb][0], d[nb][1]), yt[r][2 * nb]));
          yt[r][2 * nb + 1] = __ffma2_rn(cB, xsv[nb], __ffma2_rn(aB, make_float2(d[nb][2], d[nb][3]), yt[r][2 * nb + 1]));
        }
      }
    }
  }

  // Cross-warp reduction through shared memory (reuses the code buffer).
  __syncthreads();
  float* red = reinterpret_cast<float*>(&sm.codes[0][0][0][0]);  // [warp][token][row], 32 KB
#pragma unroll
  for (int nb = 0; nb < NB; ++nb)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int rowA = 16 * r + gid, tk0 = 2 * t4 + 8 * nb;
      red[(warp * 16 + tk0) * 64 + rowA] = yt[r][2 * nb].x;
      red[(warp * 16 + tk0 + 1) * 64 + rowA] = yt[r][2 * nb].y;
      red[(warp * 16 + tk0) * 64 + rowA + 8] = yt[r][2 * nb + 1].x;
      red[(warp * 16 + tk0 + 1) * 64 + rowA + 8] = yt[r][2 * nb + 1].y;
    }
  __syncthreads();
  const int ntk = 8 * NB;
  for (int o = tid; o < ntk * 64; o += kDecThreads) {
    const int tk = o >> 6, row = o & 63;
    const int64_t n = rb * kDecRows + row;
    if (tk < T && n < N) {
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < kDecThreads / 32; ++w) v += red[(w * 16 + tk) * 64 + row];
      if (nch == 1) Y[(int64_t)tk * N + n] = v;
      else partial[((int64_t)ch * 16 + tk) * N + n] = v;
    }
  }
  if (nch == 1) return;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int ticket = atomicAdd(&meta[1 + rb], 1);
    sm.is_last = (ticket == nch - 1);
  }
  __syncthreads();
  if (!sm.is_last) return;
  __threadfence();
  for (int o = tid; o < ntk * 64; o += kDecThreads) {
    const int tk = o >> 6, row = o & 63;
    const int64_t n = rb * kDecRows + row;
    if (tk < T && n < N) {
      float v = 0.0f;
      for (int c = 0; c < nch; ++c) v += __ldcg(&partial[((int64_t)c * 16 + tk) * N + n]);
      Y[(int64_t)tk * N + n] = v;
    }
  }
  if (tid == 0) meta[1 + rb] = 0;
}

// ---- host side -----------------------------------------------------------------------

size_t decode_ws_bytes(int64_t N, int64_t K) {
  const int64_t ngroups = K / 128;
  const int64_t nch = (ngroups + kDecGroups - 1) / kDecGroups;
  const int64_t nrb = (N + kDecRows - 1) / kDecRows;
  size_t b = 0;
  b += (size_t)ngroups * 2048 * 2;                             // Xd: 2048 * NB bytes per group, NB <= 2
  b = (b + 255) / 256 * 256;
  b += (size_t)ngroups * 16 * sizeof(float);                   // xs
  b = (b + 255) / 256 * 256;
  b += (size_t)(1 + nrb) * sizeof(int32_t);                    // meta
  b = (b + 255) / 256 * 256;
  b += (size_t)nch * 16 * (size_t)N * sizeof(float);           // partials
  return (b + 255) / 256 * 256;
}

static size_t dec_smem_bytes(int NB) {
  return kDecSmemXd + (size_t)kDecGroups * 2048 * NB + 1024;  // + 1024 for the manual alignment
}

cudaError_t launch_decode(const void* X, int T, int64_t K, const int32_t* k_t, const uint32_t* codes,
                          const uint32_t* sz, int64_t N, int S, float* Y, void* ws, cudaStream_t stream,
                          DeviceStatus* st) {
  const int64_t ngroups = K / 128;
  const int64_t nch = (ngroups + kDecGroups - 1) / kDecGroups;
  const int64_t nrb = (N + kDecRows - 1) / kDecRows;
  const int NB = T > 8 ? 2 : 1;
  uint8_t* p = static_cast<uint8_t*>(ws);
  size_t off = 0;
  uint32_t* Xd = reinterpret_cast<uint32_t*>(p + off);
  off += (size_t)ngroups * 2048 * 2;
  off = (off + 255) / 256 * 256;
  float* xs = reinterpret_cast<float*>(p + off);
  off += (size_t)ngroups * 16 * sizeof(float);
  off = (off + 255) / 256 * 256;
  int32_t* meta = reinterpret_cast<int32_t*>(p + off);
  off += (size_t)(1 + nrb) * sizeof(int32_t);
  off = (off + 255) / 256 * 256;
  float* partial = reinterpret_cast<float*>(p + off);

  CUtensorMap tm_codes, tm_sz;
  if (!make_tmap_2d(&tm_codes, codes, 4, (uint64_t)(K / 16), (uint64_t)(S * N), (uint64_t)(K / 16) * 4, 32, 64,
                    true))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tm_sz, sz, 4, (uint64_t)N, (uint64_t)(S * ngroups), (uint64_t)N * 4, 64, 8, false))
    return cudaErrorInvalidValue;

  decode_prep_kernel<<<(unsigned)ngroups, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(X), T, K, NB, k_t,
                                                             Xd, xs, meta, nrb, st);
  const size_t smem = dec_smem_bytes(NB);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nrb, (unsigned)nch);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap with the staging kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  const uint64_t lim = wait_limit();
  if (NB == 2) {
    if ((e = set_smem((const void*)decode_kernel<2>, (int)smem)) != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_kernel<2>, tm_codes, tm_sz, (const uint32_t*)Xd, (const float*)xs, k_t, meta,
                           T, N, ngroups, S, partial, Y, st, lim);
  } else {
    if ((e = set_smem((const void*)decode_kernel<1>, (int)smem)) != cudaSuccess) return e;
    e = cudaLaunchKernelEx(&cfg, decode_kernel<1>, tm_codes, tm_sz, (const uint32_t*)Xd, (const float*)xs, k_t, meta,
                           T, N, ngroups, S, partial, Y, st, lim);
  }
  if (e != cudaSuccess) return note_error("decode launch", e);
  return note_error("kernel launch", cudaGetLastError());
}

}  // namespace mobi

// ---- the decode GEMM with static scratch (mobi_gemm_decode_noalloc) -------------------
//
// For callers that cannot allocate: the decode scratch (staged activations,
// group sums, split-K tickets and partials) lives in one file-scope array of
// static device memory instead of a caller workspace. The kernels are the ones
// above; only the scratch pointer differs.

namespace mobi {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

static std::mutex g_scratch_mu;
static void* g_scratch_dev[64];

// Device address of g_decode_scratch on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
static void* noalloc_scratch(cudaError_t* err) {
  int d = 0;
  *err = cudaGetDevice(&d);
  if (*err != cudaSuccess) return nullptr;
  if (d < 0 || d >= 64) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_dev[d]) {
    void* p = nullptr;
    *err = note_error("cudaGetSymbolAddress(decode scratch)", cudaGetSymbolAddress((void**)&p, g_decode_scratch));
    if (*err != cudaSuccess) return nullptr;
    g_scratch_dev[d] = p;
  }
  return g_scratch_dev[d];
}

}  // namespace mobi

extern "C" mobi_status mobi_gemm_decode_noalloc(const void* X, int64_t T, int64_t K, const int32_t* k_t,
                                                const uint32_t* codes, const uint32_t* sz, int64_t N, int G,
                                                int S, float* Y, void* stream) {
  using namespace mobi;
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (N < 0 || K < 0 || T < 0 || S < 1 || S > 3) return MOBI_ERR_INVALID_ARG;
  if (G != 128 || K % 128 != 0 || N % 16 != 0 || T > 16 || N > (int64_t(1) << 28) || K > (int64_t(1) << 28))
    return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (T == 0 || N == 0) return MOBI_OK;
  if (K == 0) return MOBI_ERR_UNSUPPORTED_SHAPE;
  if (!X || !k_t || !codes || !sz || !Y) return MOBI_ERR_INVALID_ARG;
  if (!a16(X) || !a16(codes) || !a16(sz) || !a16(Y) || (reinterpret_cast<uintptr_t>(k_t) & 3u))
    return MOBI_ERR_MISALIGNED;
  const size_t need = decode_ws_bytes(N, K);
  if (need > kNoAllocScratchBytes) {
    char msg[128];
    snprintf(msg, sizeof msg, "decode scratch of %zu bytes exceeds the %zu-byte static array", need,
             kNoAllocScratchBytes);
    note_error(msg, cudaErrorInvalidValue);
    return MOBI_ERR_WORKSPACE;
  }
  cudaError_t e;
  DeviceStatus* st = device_status(&e);
  if (!st) return MOBI_ERR_CUDA;
  void* scratch = noalloc_scratch(&e);
  if (!scratch) return MOBI_ERR_CUDA;
  e = launch_decode(X, (int)T, K, k_t, codes, sz, N, S, Y, scratch, static_cast<cudaStream_t>(stream), st);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return MOBI_ERR_CUDA;
  }
  return MOBI_OK;
}
