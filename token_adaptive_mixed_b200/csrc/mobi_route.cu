// mobi_route.cu — MoBiRoute token routing and stable token bucketing on sm_100a.
//
// MoBiQuant explainer [ja] §2.2 / [en] §2.B: a router scores every token and
// the score decides how many residual slices it activates. Here the router is
// linear: logit_j(t) = sum_k x[t,k] Wr[k,j] + b_j and k_t = 1 + argmax_j
// (lowest j on an exact tie). Tokens are then stably sorted by k_t.
//
// route_partial_kernel: grid (token tiles of 16, K splits), 256 threads. Each
//   thread owns 8 consecutive columns per 2048-wide pass and accumulates the
//   x.Wr products of its columns in fp32; the warp reduces in fp32 and the
//   warps (and K splits) combine in fp64 in a fixed order, so the result is
//   deterministic and far more accurate than the 1e-5 near-tie band.
//   Bound: HBM read of X (T*K*2 bytes).
// bucket_kernel: one CTA. Finishes the K-split logits (if any), takes the
//   argmax, then counts and scatters the tokens in index order with warp
//   ballots, which keeps the sort stable.
// route_small_kernel (T <= 16, the decode case): both steps in one launch of
//   one thread-block cluster; see below.
#include <cstdint>

#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

constexpr int kRouteTB = 16;       // tokens per CTA
constexpr int kRouteThreads = 256;
constexpr int kRoutePass = 2048;   // columns covered per pass (256 threads x 8)

__device__ __forceinline__ int argmax_lowest(const double* l, int S) {
  int best = 0;
  for (int j = 1; j < S; ++j)
    if (l[j] > l[best]) best = j;
  return best;
}

// The same with a compile-time S, so that l stays in registers.
template <int S>
__device__ __forceinline__ int argmax_lowest_t(const double (&l)[S]) {
  int best = 0;
  double m = l[0];
#pragma unroll
  for (int j = 1; j < S; ++j)
    if (l[j] > m) { m = l[j]; best = j; }
  return best;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem)), "l"(gmem) : "memory");
}

// partial[ks][t][j] (fp64) when ksplit > 1, otherwise k_t directly.
template <int S>
__global__ void __launch_bounds__(kRouteThreads) route_partial_kernel(
    const __nv_bfloat16* __restrict__ X, int64_t T, int64_t K, const float* __restrict__ Wr,
    const float* __restrict__ bias, int64_t k_per_split, int32_t* __restrict__ k_t,
    double* __restrict__ partial) {
  __shared__ float red[kRouteThreads / 32][kRouteTB * S];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t0 = (int64_t)blockIdx.x * kRouteTB;
  const int ntok = (int)(T - t0 < kRouteTB ? T - t0 : kRouteTB);
  const int64_t kbeg = (int64_t)blockIdx.y * k_per_split;
  const int64_t kend = (K < kbeg + k_per_split) ? K : kbeg + k_per_split;

  float acc[kRouteTB][S];
#pragma unroll
  for (int i = 0; i < kRouteTB; ++i)
#pragma unroll
    for (int j = 0; j < S; ++j) acc[i][j] = 0.0f;

  for (int64_t k = kbeg + 8 * tid; k < kend; k += kRoutePass) {
    float w[8][S];
    const float* wp = Wr + k * S;
#pragma unroll
    for (int e = 0; e < 8 * S; ++e) w[e / S][e % S] = __ldg(wp + e);
#pragma unroll
    for (int i = 0; i < kRouteTB; ++i) {
      if (i < ntok) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(X + (t0 + i) * K + k));
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float x0 = bf16lo(u[p]), x1 = bf16hi(u[p]);
#pragma unroll
          for (int j = 0; j < S; ++j) {
            acc[i][j] = fmaf(x0, w[2 * p][j], acc[i][j]);
            acc[i][j] = fmaf(x1, w[2 * p + 1][j], acc[i][j]);
          }
        }
      }
    }
  }

  // Warp reduction (fp32, fixed xor tree), then warps in fp64 in order.
#pragma unroll
  for (int i = 0; i < kRouteTB; ++i)
#pragma unroll
    for (int j = 0; j < S; ++j) {
      float v = acc[i][j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][i * S + j] = v;
    }
  __syncthreads();
  if (tid < kRouteTB) {
    const int i = tid;
    if (i < ntok) {
      double l[S];
#pragma unroll
      for (int j = 0; j < S; ++j) {
        double s = 0.0;
        for (int w8 = 0; w8 < kRouteThreads / 32; ++w8) s += (double)red[w8][i * S + j];
        l[j] = s;
      }
      if (partial != nullptr) {
#pragma unroll
        for (int j = 0; j < S; ++j) partial[((int64_t)blockIdx.y * T + t0 + i) * S + j] = l[j];
      } else {
#pragma unroll
        for (int j = 0; j < S; ++j) l[j] += bias ? (double)__ldg(bias + j) : 0.0;
        k_t[t0 + i] = 1 + argmax_lowest(l, S);
      }
    }
  }
}

constexpr int kBucketThreads = 1024;

// Single CTA: optional finish of split logits, then the stable counting sort.
template <int S>
__global__ void __launch_bounds__(kBucketThreads) bucket_kernel(int64_t T, int ksplit,
                                                                const double* __restrict__ partial,
                                                                const float* __restrict__ bias,
                                                                int32_t* __restrict__ k_t,
                                                                int32_t* __restrict__ perm,
                                                                int32_t* __restrict__ offsets) {
  __shared__ int cnt[S];
  __shared__ int base[S];
  __shared__ int warp_cnt[kBucketThreads / 32][S];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  if (ksplit > 1) {
    for (int64_t t = tid; t < T; t += kBucketThreads) {
      double l[S];
#pragma unroll
      for (int j = 0; j < S; ++j) {
        double s = 0.0;
        for (int ks = 0; ks < ksplit; ++ks) s += partial[((int64_t)ks * T + t) * S + j];
        l[j] = s + (bias ? (double)bias[j] : 0.0);
      }
      k_t[t] = 1 + argmax_lowest(l, S);
    }
    __syncthreads();
    __threadfence_block();
  }

  if (tid < S) cnt[tid] = 0;
  __syncthreads();
  int local[S];
#pragma unroll
  for (int j = 0; j < S; ++j) local[j] = 0;
  for (int64_t t = tid; t < T; t += kBucketThreads) {
    const int k = k_t[t];
#pragma unroll
    for (int j = 0; j < S; ++j) local[j] += (k == j + 1);
  }
#pragma unroll
  for (int j = 0; j < S; ++j) {
    int v = local[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) atomicAdd(&cnt[j], v);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int j = 0; j < S; ++j) {
      offsets[j] = run;
      base[j] = run;
      run += cnt[j];
    }
    offsets[S] = run;
  }
  __syncthreads();

  // Stable scatter, one chunk of 1024 tokens at a time, in token order.
  for (int64_t c0 = 0; c0 < T; c0 += kBucketThreads) {
    const int64_t t = c0 + tid;
    const int k = t < T ? k_t[t] : 0;
    unsigned my_rank = 0;
#pragma unroll
    for (int j = 0; j < S; ++j) {
      const unsigned m = __ballot_sync(0xffffffffu, k == j + 1);
      if (k == j + 1) my_rank = __popc(m & ((1u << lane) - 1u));
      if (lane == 0) warp_cnt[warp][j] = __popc(m);
    }
    __syncthreads();
    if (tid < S) {  // exclusive scan over warps for value tid+1
      int run = 0;
      for (int w = 0; w < kBucketThreads / 32; ++w) {
        const int c = warp_cnt[w][tid];
        warp_cnt[w][tid] = run;
        run += c;
      }
      cnt[tid] = run;  // chunk total
    }
    __syncthreads();
    if (t < T) perm[base[k - 1] + warp_cnt[warp][k - 1] + (int)my_rank] = (int32_t)t;
    __syncthreads();
    if (tid < S) base[tid] += cnt[tid];
    __syncthreads();
  }
}

// ---- small batches (T <= 16): one launch of one 8-CTA cluster ------------------------
//
// CTA r of the cluster sums the logits of every token over its share of the
// 8-column octets of K (fp32 within a thread, fp32 xor tree within a warp,
// fp64 across warps) and stores them into CTA 0's shared memory (distributed
// shared memory); after one cluster barrier CTA 0 adds the eight partials in
// rank order (fp64), takes the argmax and writes the stable bucketing (warp
// ballots over the at most 16 tokens). The CTA's slices of X and Wr are first
// staged into shared memory with cp.async (no registers held per load, so
// every load of a pass is in flight at once), in passes of 256 octets.
// Launched as a programmatic dependent of whatever precedes it: it reads no
// global memory before griddepcontrol.wait, and lets its own dependent (the
// decode GEMM) start its set-up early.
constexpr int kRouteSmallT = 16;
constexpr int kRouteCluster = 8;
constexpr int kRoutePassOct = kRouteThreads;  // octets staged per pass: one per thread

// Dynamic shared memory of route_small_kernel<S>: X [16 tokens][pass] 16-byte
// octets, then Wr [pass][8 S] floats.
__host__ __device__ constexpr size_t route_small_smem(int S) {
  return (size_t)kRouteSmallT * kRoutePassOct * 16 + (size_t)kRoutePassOct * 8 * S * 4;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of `p` (this CTA's shared memory) in the shared memory of cluster CTA `rank`.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(p)), "r"(rank));
  return r;
}

__device__ __forceinline__ void st_dsmem_f64(uint32_t addr, double v) {
  asm volatile("st.shared::cluster.f64 [%0], %1;" ::"r"(addr), "d"(v) : "memory");
}

template <int S>
__global__ void __launch_bounds__(kRouteThreads) route_small_kernel(
    const __nv_bfloat16* __restrict__ X, int T, int64_t K, const float* __restrict__ Wr,
    const float* __restrict__ bias, int32_t* __restrict__ k_t, int32_t* __restrict__ perm,
    int32_t* __restrict__ offsets) {
  __shared__ float red[kRouteThreads / 32][kRouteSmallT * S];
  __shared__ double part[kRouteCluster][kRouteSmallT * S];  // used in CTA 0: [rank][token * S + j]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  uint32_t rank;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  const int64_t noct = K / 8;
  const int64_t o_beg = rank * noct / kRouteCluster, o_end = (rank + 1) * noct / kRouteCluster;

  extern __shared__ __align__(16) uint8_t rsm[];
  uint4* xs = reinterpret_cast<uint4*>(rsm);                                   // [token][octet]
  float* wsm = reinterpret_cast<float*>(rsm + kRouteSmallT * kRoutePassOct * 16);  // [octet][8 S]
  float acc[kRouteSmallT][S];
#pragma unroll
  for (int i = 0; i < kRouteSmallT; ++i)
#pragma unroll
    for (int j = 0; j < S; ++j) acc[i][j] = 0.0f;
  for (int64_t p0 = o_beg; p0 < o_end; p0 += kRoutePassOct) {
    const int np = (int)(o_end - p0 < kRoutePassOct ? o_end - p0 : kRoutePassOct);
    for (int i = 0; i < T; ++i)
      for (int o = tid; o < np; o += kRouteThreads)
        cp_async16(&xs[i * kRoutePassOct + o], X + (int64_t)i * K + 8 * (p0 + o));
    for (int e = tid; e < np * 2 * S; e += kRouteThreads)  // 8 S floats = 2 S pieces of 16 bytes per octet
      cp_async16(&wsm[4 * e], Wr + p0 * 8 * S + 4 * e);
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (tid < np) {
      const int o = tid;
      float w[8][S];
#pragma unroll
      for (int e = 0; e < 8 * S; ++e) w[e / S][e % S] = wsm[o * 8 * S + e];
#pragma unroll
      for (int i = 0; i < kRouteSmallT; ++i) {
        if (i < T) {
          const uint4 v = xs[i * kRoutePassOct + o];
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const float x0 = bf16lo(u[p]), x1 = bf16hi(u[p]);
#pragma unroll
            for (int j = 0; j < S; ++j) {
              acc[i][j] = fmaf(x0, w[2 * p][j], acc[i][j]);
              acc[i][j] = fmaf(x1, w[2 * p + 1][j], acc[i][j]);
            }
          }
        }
      }
    }
    __syncthreads();  // the next pass overwrites the staged slices
  }
#pragma unroll
  for (int i = 0; i < kRouteSmallT; ++i)
#pragma unroll
    for (int j = 0; j < S; ++j) {
      float v = acc[i][j];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][i * S + j] = v;
    }
  __syncthreads();
  if (tid < kRouteSmallT * S) {
    double s = 0.0;
    for (int w8 = 0; w8 < kRouteThreads / 32; ++w8) s += (double)red[w8][tid];
    st_dsmem_f64(dsmem_addr(&part[rank][tid], 0), s);
  }
  cluster_sync_all();  // every CTA's partial logits are in CTA 0's shared memory

  if (rank == 0 && warp == 0) {
    // Lane t < T: the logits of token t, partials added in rank order.
    int k = 0;
    if (lane < T) {
      double l[S];
#pragma unroll
      for (int j = 0; j < S; ++j) {
        double s = 0.0;
        for (int r = 0; r < kRouteCluster; ++r) s += part[r][lane * S + j];
        l[j] = s + (bias ? (double)__ldg(bias + j) : 0.0);
      }
      k = 1 + argmax_lowest_t<S>(l);
      k_t[lane] = k;
    }
    // Stable bucketing: tokens of value v keep their index order.
    int run = 0;
#pragma unroll
    for (int j = 0; j < S; ++j) {
      const unsigned m = __ballot_sync(0xffffffffu, k == j + 1);
      if (lane == 0) offsets[j] = run;
      if (k == j + 1) perm[run + __popc(m & ((1u << lane) - 1u))] = lane;
      run += __popc(m);
    }
    if (lane == 0) offsets[S] = run;
  }
}

template <int S>
static cudaError_t launch_route_small(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                                      int32_t* k_t, int32_t* perm, int32_t* offsets, cudaStream_t stream) {
  const size_t smem = route_small_smem(S);
  cudaError_t e = set_smem((const void*)route_small_kernel<S>, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kRouteCluster);
  cfg.blockDim = dim3(kRouteThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kRouteCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // overlap the launch with the previous kernel
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, route_small_kernel<S>, static_cast<const __nv_bfloat16*>(X), (int)T, K, Wr, bias, k_t,
                         perm, offsets);
  if (e != cudaSuccess) return note_error("route launch", e);
  return note_error("kernel launch", cudaGetLastError());
}

int route_ksplit(int64_t T, int64_t K) {
  const int64_t tiles = (T + kRouteTB - 1) / kRouteTB;
  if (tiles == 0 || tiles >= 64) return 1;
  int64_t ks = (K + 1023) / 1024;
  const int64_t want = (128 + tiles - 1) / tiles;
  if (ks > want) ks = want;
  if (ks < 1) ks = 1;
  return (int)ks;
}

size_t route_ws_bytes(int64_t T, int64_t K, int S) {
  if (T >= 1 && T <= kRouteSmallT) return 0;  // one cluster launch, no workspace
  const int ks = route_ksplit(T, K);
  return ks > 1 ? (size_t)ks * (size_t)T * (size_t)S * sizeof(double) : 0;
}

template <int S>
static cudaError_t launch_route_s(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                                  int32_t* k_t, int32_t* perm, int32_t* offsets, void* ws,
                                  cudaStream_t stream) {
  if (T >= 1 && T <= kRouteSmallT) return launch_route_small<S>(X, T, K, Wr, bias, k_t, perm, offsets, stream);
  const int ks = route_ksplit(T, K);
  int64_t kps = (K + ks - 1) / ks;
  kps = (kps + 7) / 8 * 8;  // whole 8-column octets per split
  double* partial = ks > 1 ? static_cast<double*>(ws) : nullptr;
  if (T > 0) {
    dim3 grid((unsigned)((T + kRouteTB - 1) / kRouteTB), (unsigned)ks);
    route_partial_kernel<S><<<grid, kRouteThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(X), T, K, Wr, bias, kps, k_t, partial);
  }
  bucket_kernel<S><<<1, kBucketThreads, 0, stream>>>(T, ks, partial, bias, k_t, perm, offsets);
  return note_error("kernel launch", cudaGetLastError());
}

cudaError_t launch_route(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias, int S,
                         int32_t* k_t, int32_t* perm, int32_t* offsets, void* ws, cudaStream_t stream) {
  switch (S) {
    case 1: return launch_route_s<1>(X, T, K, Wr, bias, k_t, perm, offsets, ws, stream);
    case 2: return launch_route_s<2>(X, T, K, Wr, bias, k_t, perm, offsets, ws, stream);
    default: return launch_route_s<3>(X, T, K, Wr, bias, k_t, perm, offsets, ws, stream);
  }
}

}  // namespace mobi
