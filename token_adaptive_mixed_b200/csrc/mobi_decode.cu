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
// exact A-operand values, one AND per two weights. The activations enter as
// x * 2^96 / 4^f (exact in bf16 for |x| < 2^31), so every product is
// q * x * 2^-37 exactly and every field carries the same weight. The zero
// point is folded in once per (row, group): sum_k x (q - z) = sum_k x q -
// z * sum_k x, where sum_k x comes from the same tensor-core pass with an
// all-ones code operand. fp32 accumulation happens in the tensor core
// (mma.sync m16n8k16) and in the per-group promotion
// y += scale * 2^37 * acc - scale * z * xsum.
//
// Work split (persistent, one CTA per SM). K is cut into chunks of 8 groups
// (1024 columns); a CTA owns one chunk and a contiguous range of 32-row
// blocks (two 16-row MMA tiles each). Its consumer warps form teams of four:
// the warps of a team work on the same block, each on 2 of the chunk's 8
// groups, and hand their sums to the team's first warp through shared
// memory. A warp keeps the activation fragments of its 2 groups in registers
// for the whole kernel (built once from X), which keeps its unrolled stage
// code small enough for the instruction cache. One producer warp feeds a
// TMA ring per consumer warp with (block, slice) stages, so code bytes stream
// in while earlier stages are multiplied. Chunks are combined by a second,
// programmatically dependent kernel that adds the per-chunk partials in chunk
// order (deterministic).
#include <cstdint>
#include <cstring>
#include <cstdio>
#include <mutex>

#include "../../include/mobi.h"
#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

constexpr int kDecGW = 2;                    // groups per warp (64 bytes of a code row)
constexpr int kDecQ = 4;                     // warps per team (one team per 32-row block)
constexpr int kDecChunk = kDecQ * kDecGW;    // groups per CTA chunk
constexpr int kDecRows = 32;                 // rows per stage: two 16-row MMA tiles
// A stage belongs to a team: 32 rows x the chunk's 8 groups, as two
// 128-byte-swizzled halves of 32 rows x 128 bytes, then [8 groups][32 rows]
// scale/zero words.
constexpr uint32_t kDecHalfBytes = kDecRows * 128;
constexpr uint32_t kDecSlotCodes = 2 * kDecHalfBytes;
constexpr uint32_t kDecSlotSz = kDecChunk * kDecRows * 4;
constexpr uint32_t kDecSlot = kDecSlotCodes + kDecSlotSz;  // 9 KB, a multiple of 1 KB

template <int NB>
struct DecCfg;
template <>
struct DecCfg<1> {  // T <= 8: 16 B-fragment registers per group
  static constexpr int kTeams = 3;
  static constexpr int kDepth = 6;
};
template <>
struct DecCfg<2> {  // T <= 16: 32 per group
  static constexpr int kTeams = 2;
  static constexpr int kDepth = 8;
};

template <int NB>
struct DecLayout {
  static constexpr int kWarps = kDecQ * DecCfg<NB>::kTeams;  // consumer warps; one producer warp follows
  static constexpr int kThreads = 32 * (kWarps + 1);
  // Registers per thread for one CTA: the warps are spread over the SM's four
  // 16K-register sub-partitions, so the fullest one decides.
  static constexpr int kMaxRegs = (16384 / (32 * ((kWarps + 4) / 4))) / 8 * 8 > 248
                                      ? 248
                                      : (16384 / (32 * ((kWarps + 4) / 4))) / 8 * 8;
  static constexpr int kDepth = DecCfg<NB>::kDepth;
  static constexpr int kTeams = DecCfg<NB>::kTeams;
  static constexpr uint32_t kSlots = 0;                                      // [team][slot] 9 KB, 1 KB aligned
  static constexpr uint32_t kXchg = kSlots + kTeams * kDepth * kDecSlot;     // [team][2][kDecQ-1][32][8 NB] floats
  static constexpr uint32_t kBar = kXchg + DecCfg<NB>::kTeams * 2 * (kDecQ - 1) * 32 * 8 * NB * 4;  // full, empty
  static constexpr uint32_t kReady = kBar + 2 * kTeams * kDepth * 8;  // consumers' fragments built
  static constexpr uint32_t kAbort = kReady + 8;
  static constexpr uint32_t kBytes = kAbort + 8;
  static constexpr size_t kDynamic = kBytes + 1024;  // + manual 1 KB alignment
};

constexpr float kTwo37 = 137438953472.0f;  // 2^37

__device__ __forceinline__ void mma_bf16_16816(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Exact for a power-of-two multiplier as long as nothing overflows.
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// Issue one team stage into `slot`: the chunk's 256 bytes of 32 code rows as
// two 128-byte halves (x = word column, y = s*N + row) and the matching
// [8 groups][32 rows] scale/zero words. Weights are read once per call, so
// they go in with L2 evict-first.
__device__ __forceinline__ void dec_issue(const CUtensorMap* tm_codes, const CUtensorMap* tm_sz, uint8_t* slot,
                                          uint64_t* bar, int block, int s, int N, int ngroups, int chunk,
                                          uint64_t policy) {
  mbar_arrive_expect_tx(bar, kDecSlot);
  const int y = s * N + block * kDecRows;
  tma_load_2d_hint(slot, tm_codes, chunk * kDecChunk * 8, y, bar, policy);
  tma_load_2d_hint(slot + kDecHalfBytes, tm_codes, chunk * kDecChunk * 8 + 32, y, bar, policy);
  tma_load_2d_hint(slot + kDecSlotCodes, tm_sz, block * kDecRows, s * ngroups + chunk * kDecChunk, bar, policy);
}

// Groups g0, g0 + 1 of one stage for TT tiles: four MMA chains in flight.
template <int NB, int TT>
__device__ __forceinline__ void dec_group_pair(int g0, const uint8_t* cs, const uint32_t* ss,
                                               const uint32_t (&coff)[kDecGW], const uint32_t (&B)[kDecGW][8][2 * NB],
                                               const float2 (&xs)[kDecGW][NB], const float2 (&m37)[NB],
                                               const float2 (&m1)[NB], int gid, float2 (&yA)[2][NB],
                                               float2 (&yB)[2][NB]) {
  uint2 wa[2][TT], wb[2][TT];
#pragma unroll
  for (int gg = 0; gg < 2; ++gg)
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      wa[gg][tt] = *reinterpret_cast<const uint2*>(cs + coff[g0 + gg] + tt * 16 * 128);
      wb[gg][tt] = *reinterpret_cast<const uint2*>(cs + coff[g0 + gg] + tt * 16 * 128 + 8 * 128);
    }
  float d[2][TT][NB][4];
#pragma unroll
  for (int gg = 0; gg < 2; ++gg)
#pragma unroll
    for (int tt = 0; tt < TT; ++tt)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) d[gg][tt][nb][0] = d[gg][tt][nb][1] = d[gg][tt][nb][2] = d[gg][tt][nb][3] = 0.0f;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int f = 0; f < 4; ++f) {
      const uint32_t m = 0x00030003u << (2 * f);
#pragma unroll
      for (int gg = 0; gg < 2; ++gg)
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
          const uint32_t a0 = (wa[gg][tt].x >> (8 * h)) & m, a2 = (wa[gg][tt].y >> (8 * h)) & m;
          const uint32_t a1 = (wb[gg][tt].x >> (8 * h)) & m, a3 = (wb[gg][tt].y >> (8 * h)) & m;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
            mma_bf16_16816(d[gg][tt][nb], a0, a1, a2, a3, B[g0 + gg][4 * h + f][2 * nb],
                           B[g0 + gg][4 * h + f][2 * nb + 1]);
        }
    }
#pragma unroll
  for (int gg = 0; gg < 2; ++gg) {
    const int g = g0 + gg;
    float2 xm[NB];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) xm[nb] = __fmul2_rn(xs[g][nb], m1[nb]);
#pragma unroll
    for (int tt = 0; tt < TT; ++tt) {
      const uint32_t szA = ss[g * kDecRows + tt * 16 + gid], szB = ss[g * kDecRows + tt * 16 + gid + 8];
      const float scA = __half2float(__ushort_as_half((unsigned short)(szA & 0xffffu)));
      const float zA = __half2float(__ushort_as_half((unsigned short)(szA >> 16)));
      const float scB = __half2float(__ushort_as_half((unsigned short)(szB & 0xffffu)));
      const float zB = __half2float(__ushort_as_half((unsigned short)(szB >> 16)));
      const float cA = -scA * zA, cB = -scB * zB;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        // y += m * (scale 2^37 acc - scale z xsum), as packed fp32x2 FMAs.
        yA[tt][nb] = __ffma2_rn(make_float2(cA, cA), xm[nb],
                                __ffma2_rn(__fmul2_rn(make_float2(scA, scA), m37[nb]),
                                           make_float2(d[gg][tt][nb][0], d[gg][tt][nb][1]), yA[tt][nb]));
        yB[tt][nb] = __ffma2_rn(make_float2(cB, cB), xm[nb],
                                __ffma2_rn(__fmul2_rn(make_float2(scB, scB), m37[nb]),
                                           make_float2(d[gg][tt][nb][2], d[gg][tt][nb][3]), yB[tt][nb]));
      }
    }
  }
}

// One stage: the warp's groups for TT tiles.
template <int NB, int TT>
__device__ __forceinline__ void dec_stage(int ngv, const uint8_t* cs, const uint32_t* ss,
                                          const uint32_t (&coff)[kDecGW], const uint32_t (&B)[kDecGW][8][2 * NB],
                                          const float2 (&xs)[kDecGW][NB], const float2 (&m37)[NB],
                                          const float2 (&m1)[NB], int gid, float2 (&yA)[2][NB], float2 (&yB)[2][NB]) {
  // A group beyond K has zero activations and zero-filled codes: it adds 0.
  (void)ngv;
  dec_group_pair<NB, TT>(0, cs, ss, coff, B, xs, m37, m1, gid, yA, yB);
}

// Bounded wait that also gives up once another warp has aborted.
__device__ __forceinline__ bool dec_wait(uint64_t* bar, uint32_t parity, uint64_t limit, DeviceStatus* st,
                                         uint32_t where, volatile int32_t* abort_flag) {
  for (uint64_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 255 && *abort_flag) return false;
  }
  report_error(st, kErrTimeout, where);
  *abort_flag = 1;
  return false;
}

// A group of independent problems in one launch: problem i owns the CTAs
// [cta0, cta0 + cpc * nch) of the 1-D grid, cpc CTAs per K chunk. out = Y when
// the problem has one chunk, else its per-chunk partials [chunk][T][N].
struct DecProblem {
  const __nv_bfloat16* X;
  const int32_t* k_t;
  float* out;
  int T, N, K, ngroups, nblocks, cpc, cta0;
};
// MG = table capacity: 1 for a single call (a small parameter block to copy
// per launch), kMaxGroup for a group.
template <int MG>
struct DecGroup {
  CUtensorMap tm_codes[MG];
  CUtensorMap tm_sz[MG];
  DecProblem p[MG];
  int G, S;
};

// All loop bookkeeping is incremental 32-bit arithmetic (sizes are validated
// to N, K < 2^28). Warps 0 .. kWarps-1 consume (teams of four), warp kWarps
// issues the copies.
template <int NB, int MG>
__global__ void __launch_bounds__(DecLayout<NB>::kThreads, 1) __maxnreg__(DecLayout<NB>::kMaxRegs) decode_kernel(
    const __grid_constant__ DecGroup<MG> grp, DeviceStatus* st, uint64_t limit, int early) {
  using L = DecLayout<NB>;
  constexpr int kTeams = DecCfg<NB>::kTeams;
  constexpr int kW = L::kWarps;
  constexpr int D = L::kDepth;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  // The reduction kernel behind this one may be scheduled now; it waits for
  // this grid's completion before reading anything.
  asm volatile("griddepcontrol.launch_dependents;");

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int pi = 0;  // this CTA's problem
#pragma unroll 1
  for (int i = 1; i < (MG > 1 ? grp.G : 1); ++i)
    if ((int)blockIdx.x >= grp.p[i].cta0) pi = i;
  const DecProblem& prob = grp.p[pi];
  const CUtensorMap* tm_codes = &grp.tm_codes[pi];
  const CUtensorMap* tm_sz = &grp.tm_sz[pi];
  const __nv_bfloat16* __restrict__ X = prob.X;
  const int32_t* __restrict__ k_t = prob.k_t;
  float* __restrict__ out = prob.out;
  const int T = prob.T, N = prob.N, K = prob.K, ngroups = prob.ngroups, nblocks = prob.nblocks, S = grp.S;
  const int local = (int)blockIdx.x - prob.cta0, cpc = prob.cpc;
  const int ch = local / cpc, cx = local - ch * cpc;
  // This CTA's 32-row blocks [b_begin, b_end); team t takes every kTeams-th
  // of them, starting with block b_begin + t.
  const int b_begin = (int)((int64_t)cx * nblocks / cpc);
  const int b_end = (int)((int64_t)(cx + 1) * nblocks / cpc);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBar);  // [team][slot]
  uint64_t* empty = full + kTeams * D;
  uint64_t* ready = reinterpret_cast<uint64_t*>(sm + L::kReady);
  volatile int32_t* abort_flag = reinterpret_cast<volatile int32_t*>(sm + L::kAbort);

  // One barrier per thread, then one fence per warp. A stage is freed by the
  // four warps of its team.
  for (int i = threadIdx.x; i < 2 * kTeams * D + 1; i += blockDim.x) {
    if (i < kTeams * D) mbar_init(&full[i], 1);
    else if (i < 2 * kTeams * D) mbar_init(&empty[i - kTeams * D], kDecQ);
    else mbar_init(ready, kW);
  }
  if (threadIdx.x == 0) *abort_flag = 0;
  if (lane == 0) fence_barrier_init();
  __syncthreads();
  // Launched as a programmatic dependent of the previous kernel in the
  // stream. By default nothing in global memory is read before this wait.
  // With `early` set the caller guarantees that the previous kernel writes
  // none of X, codes and sz (it is this library's routing kernel), so the
  // activations and the first weight stages are fetched before the wait and
  // only k_t is read after it.
  if (!early) asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == kW) {
    // ---------------- producer: lane w feeds team w's ring ----------------
    // All lanes poll their ring's empty barrier in one non-blocking test and
    // issue their copies together, so one poll serves every team.
    named_bar_sync(15, 32 * (kW + 1));  // the consumers' activation loads go out first
    if (lane == 0) {
      prefetch_tmap(tm_codes);
      prefetch_tmap(tm_sz);
    }
    const uint64_t policy = l2_evict_first_policy();
    const int w = lane, team = lane;
    const int myb = (w < kTeams && b_end - b_begin > team) ? (b_end - b_begin - team + kTeams - 1) / kTeams : 0;
    int r = 0, bo = 0, s = 0;  // next stage of team w: its index, block offset and slice
    // Slice 0 of the team's first block does not depend on k_t.
    if (early && myb > 0) {
      dec_issue(tm_codes, tm_sz, sm + L::kSlots + (uint32_t)(w * D) * kDecSlot, &full[w * D], b_begin + team, 0, N,
                ngroups, ch, policy);
      r = 1;
    }
    if (early) asm volatile("griddepcontrol.wait;" ::: "memory");
    int kmax = __reduce_max_sync(0xffffffffu, lane < T ? (int)__ldg(k_t + lane) : 1);
    kmax = kmax < 1 ? 1 : (kmax > S ? S : kmax);
    const int nit = myb * kmax;  // stages of team w: its blocks x slices
    if (r == 1 && ++s == kmax) { s = 0; ++bo; }
    bool gate = false;         // every consumer has built its activations
    bool ok = true;
    uint64_t idle = 0;         // polls in a row without a copy issued
    while (true) {
      // Two stages per consumer first; the rest once every consumer has its
      // activations, so that those small loads do not queue behind the rings.
      if (!gate) gate = __shfl_sync(0xffffffffu, lane == 0 ? (int)mbar_test_wait(ready, 0) : 0, 0) != 0;
      bool issued = false;
      if (ok && r < nit && (r < 2 || gate)) {
        const int slot = r % D;
        if (r < D || mbar_test_wait(&empty[w * D + slot], (uint32_t)(((r / D) & 1) ^ 1))) {
          dec_issue(tm_codes, tm_sz, sm + L::kSlots + (uint32_t)(w * D + slot) * kDecSlot, &full[w * D + slot],
                    b_begin + team + bo * kTeams, s, N, ngroups, ch, policy);
          ++r;
          if (++s == kmax) { s = 0; ++bo; }
          issued = true;
        }
      }
      if (!__any_sync(0xffffffffu, ok && r < nit)) break;
      if (__any_sync(0xffffffffu, issued)) {
        idle = 0;
      } else if (++idle >= limit || ((idle & 255) == 0 && *abort_flag)) {
        if (idle >= limit && lane == 0) {
          report_error(st, kErrTimeout, 0x2e0);
          *abort_flag = 1;
        }
        ok = false;
      }
    }
    // Normally the consumers have waited for every copy. If any warp gave up,
    // every copy issued must still land before the CTA can exit (the last
    // copy into a slot completes after the earlier ones).
    __syncwarp();
    __syncthreads();  // all consumers are done
    if (*abort_flag) {
      for (int sl = 0; sl < D && sl < r; ++sl) {
        const int last = sl + (r - 1 - sl) / D * D;
        mbar_wait(&full[w * D + sl], (uint32_t)((last / D) & 1), kDefaultWaitLimit, st, 0x2f0);
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int gid = lane >> 2, t4 = lane & 3;
  const int team = warp / kDecQ, q = warp % kDecQ;
  const int gbase = ch * kDecChunk + q * kDecGW;  // first group of this warp
  const int ngv = ngroups - gbase < 0 ? 0 : (ngroups - gbase > kDecGW ? kDecGW : ngroups - gbase);
  const int my_blocks = b_end - b_begin > team ? (b_end - b_begin - team + kTeams - 1) / kTeams : 0;
  const uint8_t* slots_t = sm + L::kSlots + (uint32_t)team * D * kDecSlot;  // the team's ring
  float* xchg = reinterpret_cast<float*>(sm + L::kXchg) + team * 2 * (kDecQ - 1) * 32 * 8 * NB;
  uint64_t* full_w = full + team * D;
  uint64_t* empty_w = empty + team * D;

  // This lane's activations (token gid + 8 nb, columns 32 t4 .. +31 of each
  // group) and k_t[lane].
  uint4 raw[kDecGW][NB][4];
#pragma unroll
  for (int g = 0; g < kDecGW; ++g)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      const int tok = gid + 8 * nb;
      if (g < ngv && tok < T) {
        const uint4* src = reinterpret_cast<const uint4*>(X + (int64_t)tok * K + (gbase + g) * 128 + 32 * t4);
#pragma unroll
        for (int v = 0; v < 4; ++v) raw[g][nb][v] = __ldg(src + v);
      } else {
#pragma unroll
        for (int v = 0; v < 4; ++v) raw[g][nb][v] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
  asm volatile("bar.arrive 15, %0;" ::"r"(32 * (kW + 1)) : "memory");

  // Activation fragments of the warp's groups, in registers for the whole
  // kernel. B[g][j][2 nb + ih] is the B fragment of k16 step j = 4h + f for
  // token gid + 8 nb: register ih holds columns 32 t4 + 16 ih + 4h + f + 8e
  // (e = 0 low half, 1 high half) of group g, scaled by 2^(96 - 2f). The
  // matching A fragment of the codes is (word 2 t4 + ih >> 8h) & (3 << 2f).
  uint32_t B[kDecGW][8][2 * NB];
  float2 xs[kDecGW][NB];  // sum_k x of tokens (2 t4, 2 t4 + 1) + 8 nb, group g
  {
    bool bad = false;
#pragma unroll
    for (int g = 0; g < kDecGW; ++g) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const uint32_t u[16] = {raw[g][nb][0].x, raw[g][nb][0].y, raw[g][nb][0].z, raw[g][nb][0].w,
                                raw[g][nb][1].x, raw[g][nb][1].y, raw[g][nb][1].z, raw[g][nb][1].w,
                                raw[g][nb][2].x, raw[g][nb][2].y, raw[g][nb][2].z, raw[g][nb][2].w,
                                raw[g][nb][3].x, raw[g][nb][3].y, raw[g][nb][3].z, raw[g][nb][3].w};
#pragma unroll
        for (int i = 0; i < 16; ++i)
          bad |= ((u[i] & 0x7F80u) >= (158u << 7)) || ((u[i] & 0x7F800000u) >= (158u << 23));
#pragma unroll
        for (int ih = 0; ih < 2; ++ih)
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const int w0 = 8 * ih + 2 * h + (f >> 1);
              const uint32_t pair = __byte_perm(u[w0], u[w0 + 4], (f & 1) ? 0x7632u : 0x5410u);
              const uint32_t e = (uint32_t)(223 - 2 * f) << 7;  // bf16 bits of 2^(96 - 2f)
              B[g][4 * h + f][2 * nb + ih] = bf16x2_mul(pair, e | (e << 16));
            }
      }
    }
    // Group sums on the tensor core: codes all 1 -> every D row is sum_k x * 2^-37.
    float d[kDecGW][NB][4];
#pragma unroll
    for (int g = 0; g < kDecGW; ++g)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) d[g][nb][0] = d[g][nb][1] = d[g][nb][2] = d[g][nb][3] = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t one = 0x00010001u << (2 * (j & 3));
#pragma unroll
      for (int g = 0; g < kDecGW; ++g)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
          mma_bf16_16816(d[g][nb], one, one, one, one, B[g][j][2 * nb], B[g][j][2 * nb + 1]);
    }
#pragma unroll
    for (int g = 0; g < kDecGW; ++g)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) xs[g][nb] = make_float2(d[g][nb][0] * kTwo37, d[g][nb][1] * kTwo37);
    if (__any_sync(0xffffffffu, bad) && lane == 0) report_error(st, kErrInputRange, 0x100);
  }
  if (lane == 0) mbar_arrive(ready);
  if (early) asm volatile("griddepcontrol.wait;" ::: "memory");
  const int my_kt = lane < T ? k_t[lane] : 0;
  int kmax = __reduce_max_sync(0xffffffffu, my_kt);
  kmax = kmax < 1 ? 1 : (kmax > S ? S : kmax);

  // k_t of the two tokens whose D columns this lane holds.
  int ktl[NB][2];
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    ktl[nb][0] = __shfl_sync(0xffffffffu, my_kt, 2 * t4 + 8 * nb);
    ktl[nb][1] = __shfl_sync(0xffffffffu, my_kt, 2 * t4 + 1 + 8 * nb);
  }

  // Code words 2 t4, 2 t4 + 1 of the warp's group g (chunk group 2q + g) of
  // row gid: in half q / 2 of the stage, 128-byte-swizzled (16-byte chunk c of
  // row r sits at c ^ (r & 7)); rows gid + 8, +16, +24 share the swizzle and
  // sit 1, 2, 3 KB further on.
  uint32_t coff[kDecGW];
#pragma unroll
  for (int g = 0; g < kDecGW; ++g)
    coff[g] = (uint32_t)(q >> 1) * kDecHalfBytes + (uint32_t)gid * 128u +
              (uint32_t)(((((q & 1) * kDecGW + g) * 2 + (t4 >> 1)) ^ gid) * 16) + (t4 & 1) * 8u;

  // y[tt][nb]: tile tt of the block, rows gid (A) and gid + 8 (B) of it,
  // tokens (2 t4, 2 t4 + 1) + 8 nb.
  float2 yA[2][NB], yB[2][NB];
#pragma unroll
  for (int tt = 0; tt < 2; ++tt)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) yA[tt][nb] = yB[tt][nb] = make_float2(0.0f, 0.0f);

  bool ok = true;
  int slot = 0;
  uint32_t parity = 0;
  int s = 0, blk = b_begin + team, blk_i = 0;
  const int total_iters = my_blocks * kmax;  // both warps of a team walk the same sequence
  for (int it = 0; it < total_iters; ++it) {
    const bool two = blk * kDecRows + 16 < N;  // the block's second tile exists (N % 16 == 0)
    if (ok) {  // every warp of the team frees each stage, also one past the last group
      const bool got = __all_sync(0xffffffffu, dec_wait(&full_w[slot], parity, limit, st, 0x200 + s, abort_flag));
      if (!got) {
        ok = false;
      } else {
        const uint8_t* cs = slots_t + (uint32_t)slot * kDecSlot;
        const uint32_t* ss = reinterpret_cast<const uint32_t*>(cs + kDecSlotCodes) + q * kDecGW * kDecRows;
        float2 m37[NB], m1[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          m37[nb] = make_float2(ktl[nb][0] > s ? kTwo37 : 0.0f, ktl[nb][1] > s ? kTwo37 : 0.0f);
          m1[nb] = make_float2(ktl[nb][0] > s ? 1.0f : 0.0f, ktl[nb][1] > s ? 1.0f : 0.0f);
        }
        // Past N the second tile holds zero-filled or neighbouring rows; its
        // sums are computed like the first tile's and never written.
        dec_stage<NB, 2>(ngv, cs, ss, coff, B, xs, m37, m1, gid, yA, yB);
        // Slot free again for the producer.
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_w[slot]);
      }
    }
    if (++slot == D) { slot = 0; parity ^= 1u; }
    if (s == kmax - 1) {
      // Team hand-off: warps 1..3 of the team pass their groups' sums to
      // warp 0, which adds them in warp order.
      float* xb = xchg + (blk_i & 1) * (kDecQ - 1) * 32 * 8 * NB;
      if (q > 0) {
        float* mine = xb + ((q - 1) * 32 + lane) * 8 * NB;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
            *reinterpret_cast<float4*>(mine + 8 * nb + 4 * tt) =
                make_float4(yA[tt][nb].x, yA[tt][nb].y, yB[tt][nb].x, yB[tt][nb].y);
      }
      named_bar_sync(1 + team, 32 * kDecQ);
      if (q == 0) {
        float* o = out + (int64_t)ch * T * N + blk * kDecRows;
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          if (tt == 1 && !two) break;
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            float v[4] = {yA[tt][nb].x, yA[tt][nb].y, yB[tt][nb].x, yB[tt][nb].y};
#pragma unroll
            for (int w = 0; w < kDecQ - 1; ++w) {
              const float4 p = *reinterpret_cast<const float4*>(xb + (w * 32 + lane) * 8 * NB + 8 * nb + 4 * tt);
              v[0] += p.x; v[1] += p.y; v[2] += p.z; v[3] += p.w;
            }
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int tk = 2 * t4 + 8 * nb + e;
              if (tk < T) {
                o[(int64_t)tk * N + tt * 16 + gid] = v[e];
                o[(int64_t)tk * N + tt * 16 + gid + 8] = v[2 + e];
              }
            }
          }
        }
      }
#pragma unroll
      for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) yA[tt][nb] = yB[tt][nb] = make_float2(0.0f, 0.0f);
      s = 0;
      blk += kTeams;
      ++blk_i;
    } else {
      ++s;
    }
  }
  // Final CTA barrier: the producer then drains its copies if a warp gave up.
  __syncwarp();
  __syncthreads();
}

// Y[t][n] = sum over chunks c (in order) of partial[c][t][n], for every problem
// of a group with more than one chunk; problem i covers the float4 indices
// [off[i], off[i + 1]) of the grid-stride range, n4 = T*N/4 of them.
// Up to 8 chunk loads are in flight at a time; the adds keep chunk order.
struct DecReduceGroup {
  const float4* partial[kMaxGroup];
  float4* Y[kMaxGroup];
  int64_t off[kMaxGroup + 1];
  int nch[kMaxGroup];
  int G;
};

__global__ void __launch_bounds__(256) decode_reduce_kernel(const __grid_constant__ DecReduceGroup grp) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const int64_t total = grp.off[grp.G];
  for (int64_t gi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; gi < total;
       gi += (int64_t)gridDim.x * blockDim.x) {
    int pi = 0;
#pragma unroll 1
    for (int j = 1; j < grp.G; ++j)
      if (gi >= grp.off[j]) pi = j;
    const int64_t i = gi - grp.off[pi], n4 = grp.off[pi + 1] - grp.off[pi];
    const int nch = grp.nch[pi];
    const float4* __restrict__ partial = grp.partial[pi];
    float4* __restrict__ Y = grp.Y[pi];
    float4 a = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int c0 = 0; c0 < nch; c0 += 8) {
      float4 b[8];
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c0 + c < nch) b[c] = __ldcg(partial + (int64_t)(c0 + c) * n4 + i);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        if (c0 + c < nch) {
          if (c0 + c == 0) a = b[c];
          else { a.x += b[c].x; a.y += b[c].y; a.z += b[c].z; a.w += b[c].w; }
        }
    }
    Y[i] = a;
  }
}

// ---- host side -----------------------------------------------------------------------

static int64_t dec_chunks(int64_t K) { return (K / 128 + kDecChunk - 1) / kDecChunk; }

size_t decode_ws_bytes(int64_t N, int64_t K) {
  const int64_t nch = dec_chunks(K);
  if (nch <= 1) return 256;
  return ((size_t)nch * 16 * (size_t)N * sizeof(float) + 255) / 256 * 256;  // partials for up to 16 tokens
}

template <int NB, int MG>
static cudaError_t launch_decode_class(const DecGroup<MG>& grp, int ctas, cudaStream_t stream, DeviceStatus* st,
                                       bool early) {
  using L = DecLayout<NB>;
  cudaError_t e = set_smem((const void*)decode_kernel<NB, MG>, (int)L::kDynamic);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)ctas);
  cfg.blockDim = dim3(L::kThreads);
  cfg.dynamicSmemBytes = L::kDynamic;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // set-up overlaps the previous kernel
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_kernel<NB, MG>, grp, st, wait_limit(), early ? 1 : 0);
  if (e != cudaSuccess) return note_error("decode launch", e);
  return note_error("kernel launch", cudaGetLastError());
}

// One launch per fragment class present (T <= 8, then 9 <= T <= 16), each a
// persistent grid of about one CTA per SM shared among that class's problems
// in proportion to their weight counts N K (at least one CTA per K chunk, at
// most one per 32-row block), then one chunk-reduction launch for every
// problem with more than one chunk. Each launch is a programmatic dependent of
// the one before; `early` as for the kernel (the launches that follow the
// first class write none of the next class's inputs).
// Fills a table of capacity MG with the problems `idx[0..n)` of one fragment
// class and launches it; problems with several chunks are appended to `red`.
template <int MG>
static cudaError_t decode_class(const DecodeJob* jobs, const int* idx, int n, int cls, int S, int sms,
                                DecReduceGroup* red, cudaStream_t stream, DeviceStatus* st, bool early) {
  double wsum = 0.0;
  for (int m = 0; m < n; ++m) wsum += (double)jobs[idx[m]].N * (double)jobs[idx[m]].K;
  DecGroup<MG> grp;
  memset(&grp, 0, sizeof grp);
  grp.G = n;
  grp.S = S;
  // CTAs per chunk: each problem's share of the SMs by weight count, rounded
  // down (at least 1, at most one per 32-row block); then the SMs left over go,
  // one chunk-width at a time, to the problem with the most weights per CTA.
  int64_t cpcs[kMaxGroup], used = 0;
  for (int m = 0; m < n; ++m) {
    const DecodeJob& j = jobs[idx[m]];
    const int64_t nch = dec_chunks(j.K), nblocks = (j.N + kDecRows - 1) / kDecRows;
    int64_t cpc = (int64_t)((double)sms * ((double)j.N * (double)j.K / wsum) / (double)nch);
    if (cpc > nblocks) cpc = nblocks;
    if (cpc < 1) cpc = 1;
    cpcs[m] = cpc;
    used += cpc * nch;
  }
  while (true) {
    int best = -1;
    double best_load = 0.0;
    for (int m = 0; m < n; ++m) {
      const DecodeJob& j = jobs[idx[m]];
      const int64_t nch = dec_chunks(j.K), nblocks = (j.N + kDecRows - 1) / kDecRows;
      if (cpcs[m] >= nblocks || used + nch > sms) continue;
      const double load = (double)j.N * (double)j.K / (double)(cpcs[m] * nch);
      if (load > best_load) { best_load = load; best = m; }
    }
    if (best < 0) break;
    ++cpcs[best];
    used += dec_chunks(jobs[idx[best]].K);
  }
  int ctas = 0;
  for (int m = 0; m < n; ++m) {
    const DecodeJob& j = jobs[idx[m]];
    const int64_t nch = dec_chunks(j.K), nblocks = (j.N + kDecRows - 1) / kDecRows;
    const int64_t cpc = cpcs[m];
    if (!make_tmap_2d(&grp.tm_codes[m], j.codes, 4, (uint64_t)(j.K / 16), (uint64_t)(S * j.N),
                      (uint64_t)(j.K / 16) * 4, 32, kDecRows, 128))
      return note_error("decode tensor map (codes)", cudaErrorInvalidValue);
    if (!make_tmap_2d(&grp.tm_sz[m], j.sz, 4, (uint64_t)j.N, (uint64_t)(S * (j.K / 128)), (uint64_t)j.N * 4,
                      kDecRows, kDecChunk, 0))
      return note_error("decode tensor map (scale/zero)", cudaErrorInvalidValue);
    grp.p[m] = DecProblem{static_cast<const __nv_bfloat16*>(j.X), j.k_t, nch > 1 ? j.partial : j.Y, j.T, (int)j.N,
                          (int)j.K, (int)(j.K / 128), (int)nblocks, (int)cpc, ctas};
    ctas += (int)(cpc * nch);
    if (nch > 1) {
      red->partial[red->G] = reinterpret_cast<const float4*>(j.partial);
      red->Y[red->G] = reinterpret_cast<float4*>(j.Y);
      red->nch[red->G] = (int)nch;
      red->off[red->G + 1] = red->off[red->G] + (int64_t)j.T * j.N / 4;
      ++red->G;
    }
  }
  return cls == 1 ? launch_decode_class<1, MG>(grp, ctas, stream, st, early)
                  : launch_decode_class<2, MG>(grp, ctas, stream, st, early);
}

// One launch per fragment class present (T <= 8, then 9 <= T <= 16), each a
// persistent grid of about one CTA per SM shared among that class's problems
// in proportion to their weight counts N K (at least one CTA per K chunk, at
// most one per 32-row block), then one chunk-reduction launch for every
// problem with more than one chunk. Each launch is a programmatic dependent of
// the one before; `early` as for the kernel (the launches that follow the
// first class write none of the next class's inputs).
cudaError_t launch_decode_grouped(const DecodeJob* jobs, int G, int S, cudaStream_t stream, DeviceStatus* st,
                                  bool early) {
  const int sms = num_sms();
  DecReduceGroup red = {};
  red.off[0] = 0;
  for (int cls = 1; cls <= 2; ++cls) {
    int idx[kMaxGroup];
    int n = 0;
    for (int i = 0; i < G; ++i) {
      const DecodeJob& j = jobs[i];
      if (j.T > 0 && j.N > 0 && (j.T > 8 ? 2 : 1) == cls) idx[n++] = i;
    }
    if (n == 0) continue;
    const cudaError_t e = n == 1 ? decode_class<1>(jobs, idx, n, cls, S, sms, &red, stream, st, early)
                                 : decode_class<kMaxGroup>(jobs, idx, n, cls, S, sms, &red, stream, st, early);
    if (e != cudaSuccess) return e;
  }
  if (red.G == 0) return cudaSuccess;

  // Chunk reduction, launched as a programmatic dependent of the decode kernel.
  int64_t blocks = (red.off[red.G] + 255) / 256;
  const int64_t cap = (int64_t)sms * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_reduce_kernel, red);
  if (e != cudaSuccess) return note_error("decode reduce launch", e);
  return note_error("kernel launch", cudaGetLastError());
}

cudaError_t launch_chunk_reduce(const float* partial, float* Y, int64_t T, int64_t N, int nch, cudaStream_t stream) {
  DecReduceGroup red = {};
  red.G = 1;
  red.partial[0] = reinterpret_cast<const float4*>(partial);
  red.Y[0] = reinterpret_cast<float4*>(Y);
  red.nch[0] = nch;
  red.off[0] = 0;
  red.off[1] = T * N / 4;
  int64_t blocks = (red.off[1] + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3(256);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_reduce_kernel, red);
  if (e != cudaSuccess) return note_error("chunk reduce launch", e);
  return note_error("kernel launch", cudaGetLastError());
}

cudaError_t launch_decode(const void* X, int T, int64_t K, const int32_t* k_t, const uint32_t* codes,
                          const uint32_t* sz, int64_t N, int S, float* Y, void* ws, cudaStream_t stream,
                          DeviceStatus* st, bool early) {
  const DecodeJob job{X, k_t, codes, sz, Y, static_cast<float*>(ws), N, K, T};
  return launch_decode_grouped(&job, 1, S, stream, st, early);
}

}  // namespace mobi

// ---- the decode GEMM with static scratch (mobi_gemm_decode_noalloc) -------------------
//
// For callers that cannot allocate: the decode scratch (the per-chunk fp32
// partial sums [chunk][T][N] for up to 16 tokens, used when K spans more than
// one 1024-column chunk) lives in one file-scope array of static device memory
// instead of a caller workspace. The kernels are the ones above; only the
// scratch pointer differs.

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
  clear_message();
  auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (N < 0 || K < 0 || T < 0 || S < 1 || S > kMaxSlices) return MOBI_ERR_INVALID_ARG;
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
    note_message(msg);
    return MOBI_ERR_WORKSPACE;
  }
  cudaError_t e;
  DeviceStatus* st = device_status(&e);
  if (!st) return status_of(e);
  void* scratch = noalloc_scratch(&e);
  if (!scratch) return status_of(e);
  return status_of(
      launch_decode(X, (int)T, K, k_t, codes, sz, N, S, Y, scratch, static_cast<cudaStream_t>(stream), st, false));
}
