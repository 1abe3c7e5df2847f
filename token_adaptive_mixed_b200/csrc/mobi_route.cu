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

// Cluster c of the grid routes problem c of the group (one call is a group of one).
template <int S, int MG>
__global__ void __launch_bounds__(kRouteThreads) route_small_kernel(const __grid_constant__ RouteSmallGroupT<MG> grp) {
  __shared__ float red[kRouteThreads / 32][kRouteSmallT * S];
  __shared__ double part[kRouteCluster][kRouteSmallT * S];  // used in CTA 0: [rank][token * S + j]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const RouteSmallProblem& prob = grp.p[MG > 1 ? blockIdx.x / kRouteCluster : 0];
  const __nv_bfloat16* __restrict__ X = prob.X;
  const float* __restrict__ Wr = prob.Wr;
  const float* __restrict__ bias = prob.bias;
  int32_t* __restrict__ k_t = prob.k_t;
  int32_t* __restrict__ perm = prob.perm;
  int32_t* __restrict__ offsets = prob.offsets;
  const int64_t K = prob.K;
  const int T = prob.T;
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

template <int S, int MG>
static cudaError_t launch_route_small_group(const RouteSmallGroupT<MG>& grp, cudaStream_t stream) {
  const size_t smem = route_small_smem(S);
  cudaError_t e = set_smem((const void*)route_small_kernel<S, MG>, (int)smem);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kRouteCluster * grp.G);
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
  e = cudaLaunchKernelEx(&cfg, route_small_kernel<S, MG>, grp);
  if (e != cudaSuccess) return note_error("route launch", e);
  return note_error("kernel launch", cudaGetLastError());
}

template <int S>
static cudaError_t launch_route_small(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                                      int32_t* k_t, int32_t* perm, int32_t* offsets, cudaStream_t stream) {
  RouteSmallGroupT<1> grp = {};
  grp.G = 1;
  grp.p[0] = RouteSmallProblem{static_cast<const __nv_bfloat16*>(X), Wr, bias, k_t, perm, offsets, K, (int)T};
  return launch_route_small_group<S, 1>(grp, stream);
}

// Routing of a group of small batches (every T <= 16, same S), one cluster each.
cudaError_t launch_route_small_grouped(const RouteSmallGroup& grp, int S, cudaStream_t stream) {
  switch (S) {
    case 1: return launch_route_small_group<1, kMaxGroup>(grp, stream);
    case 2: return launch_route_small_group<2, kMaxGroup>(grp, stream);
    case 3: return launch_route_small_group<3, kMaxGroup>(grp, stream);
    default: return launch_route_small_group<4, kMaxGroup>(grp, stream);
  }
}

// ---- threshold routing with a two-layer MLP scorer -----------------------------------
//
// MoBiQuant explainer [ja] §2.2 (a 2-layer MLP scores each token; at inference
// a threshold turns the gate into a binary mask, and moving the threshold sets
// how many slices are active) and [en] §2.B ("Differentiable Gating",
// "Dynamic Adjustment": a larger delta activates fewer slices). Readings: ReLU
// hidden layer, one score per residual slice, slice j+1 active iff
// sigmoid(score_j / tau) > delta (i.e. score_j > tau * log(delta / (1 - delta))),
// k_t = 1 + the number of active residual slices.
//
// route_mlp_hidden_kernel<TT>: the first layer's pre-activations, split along
//   K: P[s][t][i] = sum_{k in split s} x[t,k] W1[k,i] (fp32 FMAs in k order).
//   CTA = 16 TT tokens x 128 hidden units, 256 threads, each TT tokens x 8
//   units (columns 4 tx .. 4 tx + 3 and 64 + 4 tx .. 64 + 4 tx + 3, so the
//   128-bit shared loads of a quarter-warp hit distinct banks); K runs in
//   32-row chunks: W1 double-buffered through cp.async, the x chunk prefetched
//   in registers and stored k-major as fp32. TT = 8 (an 8 x 8 register tile,
//   64 FMAs per 4 shared loads) from 512 tokens on, where the layer is
//   ALU-bound (T K H FMAs); TT = 4 below; TT = 1 up to 16 tokens, where it is
//   bound by the W1 read (K H 4 bytes).
// route_mlp_score_kernel<S>: one CTA of 128 threads per token: h_i =
//   max(0, sum_s P[s][t][i] + b1[i]) (splits in order), the thread's products
//   h_i W2[i][j] accumulated over i = tid, tid + 128, ..., an xor tree per warp
//   and the four warps in order, + b2[j], compared with the threshold in fp64.
// The bucketing is bucket_kernel (no split logits).
constexpr int kMlpHidTile = 128, kMlpKc = 32, kMlpThreads = 256, kMlpScoreThreads = 128;
constexpr int kMlpMinSplitK = 64;

template <int TT>
__global__ void __launch_bounds__(kMlpThreads, 2) route_mlp_hidden_kernel(const __nv_bfloat16* __restrict__ X,
                                                                         int64_t T, int64_t K,
                                                                         const float* __restrict__ W1, int64_t H,
                                                                         int64_t k_per_split,
                                                                         float* __restrict__ P) {
  constexpr int kTok = 16 * TT;
  constexpr int kXPieces = kTok * kMlpKc / 8;  // 8-bf16 pieces of x per chunk
  constexpr int kXPer = (kXPieces + kMlpThreads - 1) / kMlpThreads;  // per thread
  constexpr int kXPad = TT == 8 ? 0 : 4;       // row padding (none at TT = 8: 48 KB of static shared memory)
  __shared__ __align__(16) float xs[kMlpKc][kTok + kXPad];       // k-major fp32 copy of the x chunk
  __shared__ __align__(16) float wsm[2][kMlpKc][kMlpHidTile];    // W1 chunks, double-buffered
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int64_t t0 = (int64_t)blockIdx.x * kTok, h0 = (int64_t)blockIdx.y * kMlpHidTile;
  const int64_t split = blockIdx.z, kb = split * k_per_split;
  const int64_t ke = kb + k_per_split < K ? kb + k_per_split : K;
  const bool vec = (H & 3) == 0 && (reinterpret_cast<uintptr_t>(W1) & 15) == 0;

  // W1 rows [k0, k0 + 32) x columns [h0, h0 + 128) into wsm[buf]: cp.async when
  // every 16-byte piece is aligned, else plain loads; columns >= H read as 0.
  auto stage_w = [&](int buf, int64_t k0) {
#pragma unroll
    for (int m = 0; m < kMlpKc * kMlpHidTile / 4 / kMlpThreads; ++m) {
      const int e = tid + m * kMlpThreads, r = e >> 5, c4 = (e & 31) * 4;
      const int64_t h = h0 + c4;
      const float* src = W1 + (k0 + r) * H + h;
      float* dst = &wsm[buf][r][c4];
      if (vec && h < H) {  // H % 4 == 0, so h + 3 < H
        cp_async16(dst, src);
      } else {
        dst[0] = h < H ? __ldg(src) : 0.0f;
        dst[1] = h + 1 < H ? __ldg(src + 1) : 0.0f;
        dst[2] = h + 2 < H ? __ldg(src + 2) : 0.0f;
        dst[3] = h + 3 < H ? __ldg(src + 3) : 0.0f;
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  // Piece e of a chunk: token row e / 4, columns 8 (e % 4) .. +7.
  auto load_x = [&](int64_t k0, uint4 (&v)[kXPer]) {
#pragma unroll
    for (int m = 0; m < kXPer; ++m) {
      const int e = tid + m * kMlpThreads, xr = e >> 2, xc = (e & 3) * 8;
      v[m] = make_uint4(0u, 0u, 0u, 0u);
      if (e < kXPieces && t0 + xr < T) v[m] = __ldg(reinterpret_cast<const uint4*>(X + (t0 + xr) * K + k0 + xc));
    }
  };
  auto store_x = [&](const uint4 (&v)[kXPer]) {
#pragma unroll
    for (int m = 0; m < kXPer; ++m) {
      const int e = tid + m * kMlpThreads, xr = e >> 2, xc = (e & 3) * 8;
      if (e < kXPieces) {
        const uint32_t w[4] = {v[m].x, v[m].y, v[m].z, v[m].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // bf16 -> fp32 is a 16-bit shift
          xs[xc + 2 * q][xr] = __uint_as_float(w[q] << 16);
          xs[xc + 2 * q + 1][xr] = __uint_as_float(w[q] & 0xffff0000u);
        }
      }
    }
  };

  float acc[TT][8];
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

  // K and every split are multiples of 32, so each split is a whole number of chunks.
  uint4 xv_next[kXPer];
  load_x(kb, xv_next);
  stage_w(0, kb);
  int buf = 0;
  for (int64_t k0 = kb; k0 < ke; k0 += kMlpKc, buf ^= 1) {
    store_x(xv_next);  // xs is free: the previous chunk ended with a barrier
    if (k0 + kMlpKc < ke) {
      load_x(k0 + kMlpKc, xv_next);
      stage_w(buf ^ 1, k0 + kMlpKc);  // wsm[buf ^ 1] is free for the same reason
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kMlpKc; ++c) {
      float xv[TT];
      if constexpr (TT == 4) {
        const float4 q = *reinterpret_cast<const float4*>(&xs[c][ty * 4]);
        xv[0] = q.x; xv[1] = q.y; xv[2] = q.z; xv[3] = q.w;
      } else if constexpr (TT == 8) {
        const float4 q0 = *reinterpret_cast<const float4*>(&xs[c][ty * 8]);
        const float4 q1 = *reinterpret_cast<const float4*>(&xs[c][ty * 8 + 4]);
        xv[0] = q0.x; xv[1] = q0.y; xv[2] = q0.z; xv[3] = q0.w;
        xv[4] = q1.x; xv[5] = q1.y; xv[6] = q1.z; xv[7] = q1.w;
      } else {
#pragma unroll
        for (int i = 0; i < TT; ++i) xv[i] = xs[c][ty * TT + i];
      }
      const float4 wa = *reinterpret_cast<const float4*>(&wsm[buf][c][tx * 4]);
      const float4 wb = *reinterpret_cast<const float4*>(&wsm[buf][c][64 + tx * 4]);
      const float w[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
      for (int i = 0; i < TT; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(xv[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
  asm volatile("griddepcontrol.launch_dependents;");
#pragma unroll
  for (int i = 0; i < TT; ++i) {
    const int64_t t = t0 + ty * TT + i;
    if (t >= T) continue;
    float* row = P + (split * T + t) * H;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int64_t h = h0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (h < H) row[h] = acc[i][j];
    }
  }
}

template <int S>
__global__ void __launch_bounds__(kMlpScoreThreads) route_mlp_score_kernel(const float* __restrict__ P, int64_t T,
                                                                          int64_t H, int ksplit,
                                                                          const float* __restrict__ b1,
                                                                          const float* __restrict__ W2,
                                                                          const float* __restrict__ b2,
                                                                          double thr, int32_t* __restrict__ k_t) {
  constexpr int J = S - 1;
  __shared__ float red[kMlpScoreThreads / 32][J];
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  float acc[J];
#pragma unroll
  for (int j = 0; j < J; ++j) acc[j] = 0.0f;
  for (int64_t i = tid; i < H; i += kMlpScoreThreads) {
    float pre = 0.0f;
    const float* p = P + t * H + i;
    const int64_t stride = T * H;
    int sp = 0;
    for (; sp + 8 <= ksplit; sp += 8) {  // eight loads in flight, then the adds in split order
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = p[(int64_t)(sp + u) * stride];
#pragma unroll
      for (int u = 0; u < 8; ++u) pre += v[u];
    }
    for (; sp < ksplit; ++sp) pre += p[(int64_t)sp * stride];
    const float hv = fmaxf(pre + (b1 ? __ldg(b1 + i) : 0.0f), 0.0f);
#pragma unroll
    for (int j = 0; j < J; ++j) acc[j] = fmaf(hv, __ldg(W2 + i * J + j), acc[j]);
  }
#pragma unroll
  for (int j = 0; j < J; ++j) {
    float v = acc[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp][j] = v;
  }
  __syncthreads();
  if (tid == 0) {
    int active = 0;
#pragma unroll
    for (int j = 0; j < J; ++j) {
      float v = red[0][j];
#pragma unroll
      for (int w = 1; w < kMlpScoreThreads / 32; ++w) v += red[w][j];
      if (b2) v += __ldg(b2 + j);
      active += ((double)v > thr) ? 1 : 0;
    }
    k_t[t] = 1 + active;
  }
}

__global__ void route_mlp_base_only_kernel(int64_t T, int32_t* __restrict__ k_t) {
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) k_t[t] = 1;
}

// Splits of K for the hidden layer: as many as fit one wave of two CTAs per SM
// (no partial second wave), each split a multiple of 32 rows and at least 64.
// Tokens per CTA tile: 16 (one per thread row) up to 16 tokens, 64 below 512,
// 128 (an 8 x 8 register tile per thread) from there on.
static int mlp_tt(int64_t T) { return T <= 16 ? 1 : (T < 512 ? 4 : 8); }

static int64_t mlp_k_per_split(int64_t T, int64_t K, int64_t H, int sms) {
  const int64_t tok = 16 * mlp_tt(T);
  int64_t base = ((T + tok - 1) / tok) * ((H + kMlpHidTile - 1) / kMlpHidTile);
  if (base < 1) base = 1;
  int64_t ks = 2 * (int64_t)sms / base;
  const int64_t kmax = K / kMlpMinSplitK > 0 ? K / kMlpMinSplitK : 1;
  if (ks > kmax) ks = kmax;
  if (ks < 1) ks = 1;
  int64_t kps = (K + ks - 1) / ks;
  kps = (kps + kMlpKc - 1) / kMlpKc * kMlpKc;
  return kps > 0 ? kps : kMlpKc;
}

size_t route_mlp_ws_bytes(int64_t T, int64_t K, int64_t H, int sms) {
  if (T <= 0 || H <= 0) return 0;
  const int64_t kps = mlp_k_per_split(T, K, H, sms);
  const int64_t ks = K > 0 ? (K + kps - 1) / kps : 1;
  return ((size_t)ks * (size_t)T * (size_t)H * sizeof(float) + 255) / 256 * 256;
}

template <int S>
static void launch_mlp_score(const float* P, int64_t T, int64_t H, int ks, const float* b1, const float* W2,
                             const float* b2, double thr, int32_t* k_t, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)T);
  cfg.blockDim = dim3(kMlpScoreThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaLaunchKernelEx(&cfg, route_mlp_score_kernel<S>, P, T, H, ks, b1, W2, b2, thr, k_t);
}

cudaError_t launch_route_mlp(const void* X, int64_t T, int64_t K, const float* W1, const float* b1, int64_t H,
                             const float* W2, const float* b2, int S, double thr, int32_t* k_t, int32_t* perm,
                             int32_t* offsets, void* ws, cudaStream_t stream, int sms) {
  if (T > 0 && S == 1) {  // no residual slice to score: every token keeps the base slice only
    route_mlp_base_only_kernel<<<(unsigned)((T + 255) / 256), 256, 0, stream>>>(T, k_t);
  } else if (T > 0) {
    float* P = static_cast<float*>(ws);
    const int64_t kps = mlp_k_per_split(T, K, H, sms);
    const int ks = (int)((K + kps - 1) / kps);
    const int tt = mlp_tt(T);
    const int64_t tok = 16 * tt;
    dim3 grid((unsigned)((T + tok - 1) / tok), (unsigned)((H + kMlpHidTile - 1) / kMlpHidTile), (unsigned)ks);
    const __nv_bfloat16* Xb = static_cast<const __nv_bfloat16*>(X);
    if (tt == 1)
      route_mlp_hidden_kernel<1><<<grid, kMlpThreads, 0, stream>>>(Xb, T, K, W1, H, kps, P);
    else if (tt == 4)
      route_mlp_hidden_kernel<4><<<grid, kMlpThreads, 0, stream>>>(Xb, T, K, W1, H, kps, P);
    else
      route_mlp_hidden_kernel<8><<<grid, kMlpThreads, 0, stream>>>(Xb, T, K, W1, H, kps, P);
    if (S == 2)
      launch_mlp_score<2>(P, T, H, ks, b1, W2, b2, thr, k_t, stream);
    else if (S == 3)
      launch_mlp_score<3>(P, T, H, ks, b1, W2, b2, thr, k_t, stream);
    else
      launch_mlp_score<4>(P, T, H, ks, b1, W2, b2, thr, k_t, stream);
  }
  switch (S) {
    case 1: bucket_kernel<1><<<1, kBucketThreads, 0, stream>>>(T, 1, nullptr, nullptr, k_t, perm, offsets); break;
    case 2: bucket_kernel<2><<<1, kBucketThreads, 0, stream>>>(T, 1, nullptr, nullptr, k_t, perm, offsets); break;
    case 3: bucket_kernel<3><<<1, kBucketThreads, 0, stream>>>(T, 1, nullptr, nullptr, k_t, perm, offsets); break;
    default: bucket_kernel<4><<<1, kBucketThreads, 0, stream>>>(T, 1, nullptr, nullptr, k_t, perm, offsets); break;
  }
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
    case 3: return launch_route_s<3>(X, T, K, Wr, bias, k_t, perm, offsets, ws, stream);
    default: return launch_route_s<4>(X, T, K, Wr, bias, k_t, perm, offsets, ws, stream);
  }
}

}  // namespace mobi
