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
// Work split (persistent, one CTA per SM, stream-K style). K is cut into
// chunks of 8 groups (1024 columns). Once k_t is known (the slices each
// problem reads), the 16-row tiles of all (problem, chunk) pairs are laid out
// in one sequence, each costing its slices x (groups + a per-stage overhead),
// and every CTA takes the tiles whose start falls in its equal share of the
// total cost. A CTA's range is one or a few segments (runs of tiles in one
// chunk). For each segment the CTA builds the chunk's B operand image in
// shared memory (read with ldmatrix), then its warps split the segment's
// (tile, slice) stages evenly, one contiguous run each; every warp streams its
// stages' codes and scale/zero words through its own TMA ring (it issues its
// own copies and waits on its own barriers). A tile
// is cut between two warps only before its last slice: the second warp leaves
// that slice's sums in shared memory and the first adds them after the
// segment's barrier, which rounds exactly as the uncut order does. Chunks
// are combined by a second, programmatically dependent kernel that adds the
// per-chunk partials in chunk order (deterministic).
#include <cstdint>
#include <cstring>
#include <cstdio>
#include <mutex>

#include "../../include/mobi.h"
#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

constexpr int kDecChunk = 8;       // groups per K chunk (1024 columns)
constexpr int kDecRows = 16;       // rows per tile (one m16n8k16 A tile)
// Warps per CTA and stages per warp ring, per fragment class. T <= 8 runs 16
// warps (128 registers each) with two-stage rings; T <= 16 needs more
// registers per warp and runs 12 with three-stage rings. Both load the B
// fragments two k16 steps at a time, just before their MMAs; T <= 16 also
// reads the group sums from shared memory at each promotion.
template <int NB>
struct DecCfg {
  static constexpr int kWarps = NB == 1 ? 16 : 12;
  static constexpr int kDepth = NB == 1 ? 2 : 3;
  static constexpr bool kJitB = true;
  static constexpr bool kXsSmem = NB != 1;
};
constexpr int kDecStageOv = 3;     // fixed cost of a stage, in groups (work split cost model)
constexpr int kDecSegCost = 28 * (kDecChunk + kDecStageOv);  // set-up of a segment: about 28 full stages
// A stage is one (tile, slice): the chunk's 8 groups of 16 code rows as two
// 128-byte-swizzled halves of 16 rows x 128 bytes (4 KB, 1 KB aligned), and
// the [8 groups][16 rows] scale/zero words (512 bytes, in a ring of their own).
constexpr uint32_t kDecHalf = kDecRows * 128;
constexpr uint32_t kDecCodes = 2 * kDecHalf;
constexpr uint32_t kDecSz = kDecChunk * kDecRows * 4;

// Shared memory of the decode kernel for NB 8-token column blocks (T <= 8 NB).
template <int NB>
struct DecLayout {
  static constexpr int kWarps = DecCfg<NB>::kWarps;
  static constexpr int kDepth = DecCfg<NB>::kDepth;
  static constexpr int kThreads = 32 * kWarps;
  static constexpr uint32_t kCodes = 0;                                          // [warp][depth] code stages
  static constexpr uint32_t kSzs = kCodes + kWarps * kDepth * kDecCodes;         // [warp][depth] scale/zero stages
  static constexpr uint32_t kBimg = kSzs + kWarps * kDepth * kDecSz;             // B image, 16 KB per NB
  static constexpr uint32_t kBimgBytes = kDecChunk * NB * 8 * 256;
  static constexpr uint32_t kXs = kBimg + kBimgBytes;                            // sum_k x [group][16 tokens]
  static constexpr uint32_t kSc = kXs + kDecChunk * 16 * 4;                      // [warp][group][row] float2
  static constexpr uint32_t kHead = kSc + kWarps * kDecChunk * kDecRows * 8;     // [warp][nb][A/B][lane] float2
  static constexpr uint32_t kBar = kHead + kWarps * NB * 2 * 32 * 8;             // [warp][depth] full barriers
  static constexpr uint32_t kNever = kBar + kWarps * kDepth * 8;                 // a barrier nothing completes
  static constexpr uint32_t kBytes = kNever + 8;
  static constexpr size_t kDynamic = kBytes + 1024;  // + manual 1 KB alignment
  static_assert(kDynamic <= 232448, "fits the opt-in shared memory of one CTA");
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

// The same with a zero accumulator: d = A B.
__device__ __forceinline__ void mma_bf16_16816_z(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                 uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(0.0f));
}

// Four 8x8 b16 matrices: lane l gives the address of row l % 8 of matrix l / 8.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Issue one stage: the codes of 16-row tile `tile`, slice s, chunk `chunk`
// (x = word column, y = the code map's row: s N + row when one map covers
// every slice, the row alone with one map per slice) and its scale/zero
// words. 2-bit codes fill two 2 KB halves (64 words per row and chunk), 1-bit
// codes one (32 words).
__device__ __forceinline__ void dec_issue(const CUtensorMap* tm_codes, const CUtensorMap* tm_sz, uint8_t* codes,
                                          uint8_t* sz, uint64_t* bar, int y, int bits, int tile, int s,
                                          int ngroups, int chunk, uint64_t policy) {
  mbar_arrive_expect_tx(bar, kDecHalf * bits + kDecSz);
  tma_load_2d_hint(codes, tm_codes, chunk * kDecChunk * 4 * bits, y, bar, policy);
  if (bits == 2) tma_load_2d_hint(codes + kDecHalf, tm_codes, chunk * kDecChunk * 8 + 32, y, bar, policy);
  tma_load_2d_hint(sz, tm_sz, tile * kDecRows, s * ngroups + chunk * kDecChunk, bar, policy);
}

// Bounded wait; records the site and returns false when the limit runs out.
// A test-sized limit (mobi_debug_set_wait_limit below 64) polls without the
// hardware suspension of try_wait, so that a stage still in flight runs it out.
__device__ __forceinline__ bool dec_wait(uint64_t* bar, uint32_t parity, uint64_t limit, DeviceStatus* st,
                                         uint32_t where) {
  if (limit < 64) {
    for (uint64_t i = 0; i < limit; ++i)
      if (mbar_test_wait(bar, parity)) return true;
  } else {
    for (uint64_t i = 0; i < limit; ++i)
      if (mbar_try_wait(bar, parity)) return true;
  }
  report_error(st, kErrTimeout, where);
  return false;
}

// One problem of a launch: nblocks 16-row tiles, nch K chunks. out = Y when
// the problem has one chunk, else its per-chunk partials [chunk][T][N].
struct DecProblem {
  const __nv_bfloat16* X;
  const int32_t* k_t;
  float* out;
  int T, N, K, ngroups, nblocks, nch;
};
// MG = table capacity: 1 for a single call (a small parameter block to copy
// per launch), kMaxGroup for a group.
// BITS: 2 or 1 (every slice that wide, one code map per problem over all
// slices) or 3 (slice widths given by mask1: bit s set = slice s is 1-bit;
// one code map per slice).
template <int MG, int BITS = 2>
struct DecGroup {
  static constexpr int kMaps = BITS == 3 ? kMaxSlices : 1;
  CUtensorMap tm_codes[MG][kMaps];
  CUtensorMap tm_sz[MG];
  DecProblem p[MG];
  int G, S;
  int mask1;
};

// The cost terms of the work split, per problem: a tile of a full chunk costs
// u_full = k_max (8 + ov), a tile of the last chunk u_last = k_max (g_last +
// ov) (the stages it reads, each its groups plus a fixed overhead), and every
// chunk starts with the set-up cost Z of a segment (its B image), paid by the
// CTA whose range crosses into it; problem m starts at pre[m] of the sequence,
// pre[G] is the total.
template <int MG>
struct DecSplit {
  long long pre[MG + 1];
  long long chunk[MG];  // cost of one full chunk: Z + tiles x u_full
  int u_full[MG], u_last[MG], km[MG];
};

// Warp 0, one lane per problem. Every CTA computes the same terms (the same
// integer operations on the same k_t), so no CTA waits for another.
template <int MG, int BITS>
__device__ __forceinline__ void dec_split(const DecGroup<MG, BITS>& grp, int lane, DecSplit<MG>* sp) {
  const int G = MG > 1 ? grp.G : 1;
  long long w = 0;
  if (lane < G) {
    const DecProblem& pr = grp.p[lane];
    int km = 1;
    for (int t = 0; t < pr.T && t < 16; ++t) km = max(km, (int)pr.k_t[t]);
    km = km > grp.S ? grp.S : km;  // at least 1, at most S, as the stages clamp it
    const int g_last = pr.ngroups - (pr.nch - 1) * kDecChunk;
    const int uf = km * (kDecChunk + kDecStageOv), ul = km * (g_last + kDecStageOv);
    const long long cf = kDecSegCost + (long long)pr.nblocks * uf;
    w = cf * (pr.nch - 1) + kDecSegCost + (long long)pr.nblocks * ul;
    sp->km[lane] = km;
    sp->u_full[lane] = uf;
    sp->u_last[lane] = ul;
    sp->chunk[lane] = cf;
  }
  long long pre = w;  // inclusive prefix over the problems
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, pre, o);
    if (lane >= o) pre += v;
  }
  if (lane < G) sp->pre[lane] = pre - w;
  if (lane == G - 1) sp->pre[G] = pre;
}

// The B image of the chunk: for group g, k16 step j = 4h + f, column block nb
// (tokens 8 nb .. 8 nb + 7) and half m, an 8 x 8 b16 matrix whose row n holds,
// at column c = 2 t4 + e, x[8 nb + n][128 g + 32 t4 + 16 m + 4h + f + 8e]
// scaled by 2^(96 - 2f) (exact in bf16 for |x| < 2^31). ldmatrix of (j, m = 0)
// and (j, m = 1) gives exactly the B fragment that pairs with the A fragment
// `(word >> 8h) & (0x00030003 << 2f)` of words 2 t4, 2 t4 + 1. Matrices are
// 128 bytes each, [g][nb][j][m] in order, so one ldmatrix.x4 reads two steps.
__device__ __forceinline__ uint32_t bimg_off(int g, int nb, int j, int m, int NB) {
  return ((((uint32_t)g * NB + nb) * 8 + j) * 2 + m) * 128u;
}

// A warp boundary in a segment's stage sequence (stage x = tile x / km, slice
// x % km), moved to the nearest place where a tile is either not cut or cut
// just before its last slice. The warp that holds the tile's other slices then
// finishes it with one add of the last slice's masked sums, the same rounding
// as the uncut sequence: results do not depend on the split. Runs of at least
// km stages stay non-empty (a boundary moves by at most one stage).
__device__ __forceinline__ int dec_cut(int x, int km) {
  const int o = x % km;
  if (o == 0 || o == km - 1) return x;
  return 2 * o <= km - 1 ? x - o : x - o + km - 1;
}

// Code width of slice s (2 or 1 bits) for a launch of width mode BITS.
template <int BITS>
__device__ __forceinline__ int dec_width(int mask1, int s) {
  return BITS == 3 ? (((mask1 >> s) & 1) ? 1 : 2) : BITS;
}

// Tile sums of one warp for 16 rows (gid, gid + 8) and the lane's tokens
// 8 nb + 2 t4 + {0, 1}, written to o[t N + row] for tokens < T.
template <int NB>
__device__ __forceinline__ void dec_write_tile(float* o, int T, int N, int gid, int t4, const float2* yA,
                                               const float2* yB) {
#pragma unroll
  for (int nb = 0; nb < NB; ++nb) {
    const int t0 = 8 * nb + 2 * t4;
    if (t0 < T) {
      o[(int64_t)t0 * N + gid] = yA[nb].x;
      o[(int64_t)t0 * N + gid + 8] = yB[nb].x;
    }
    if (t0 + 1 < T) {
      o[(int64_t)(t0 + 1) * N + gid] = yA[nb].y;
      o[(int64_t)(t0 + 1) * N + gid + 8] = yB[nb].y;
    }
  }
}

// All loop bookkeeping is 32-bit arithmetic (sizes are validated to N, K <
// 2^28); positions in the cost sequence are 64-bit.
template <int NB, int MG, int BITS>
__global__ void __launch_bounds__(DecLayout<NB>::kThreads, 1) decode_kernel(
    const __grid_constant__ DecGroup<MG, BITS> grp, DeviceStatus* st, uint64_t limit) {
  using L = DecLayout<NB>;
  constexpr int D = L::kDepth;
  constexpr int kDecWarps = L::kWarps;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ DecSplit<MG> sp;
  __shared__ int s_abort;
  __shared__ float* s_tail_o[kDecWarps];  // where each warp's unfinished tile goes, and its T, N
  __shared__ int2 s_tail_tn[kDecWarps];

  // The reduction kernel behind this one may be scheduled now; it waits for
  // this grid's completion before reading anything.
  asm volatile("griddepcontrol.launch_dependents;");
  // Launched as a programmatic dependent of the previous kernel: nothing in
  // global memory is read before this wait (the split needs k_t).
  asm volatile("griddepcontrol.wait;" ::: "memory");

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gid = lane >> 2, t4 = lane & 3;
  const int G = MG > 1 ? grp.G : 1;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L::kBar) + warp * D;
  uint64_t* never = reinterpret_cast<uint64_t*>(sm + L::kNever);
  if (warp == 0) dec_split(grp, lane, &sp);
  if (threadIdx.x == 32) s_abort = 0;
  if (lane == 0) {
    for (int d = 0; d < D; ++d) mbar_init(&full[d], 1);
    if (warp == 0) mbar_init(never, 1);
    fence_barrier_init();
  }
  __syncthreads();

  // This CTA's share of the cost sequence: the tiles starting in [X0, X1).
  const long long Wt = sp.pre[G], C = gridDim.x, bi = blockIdx.x;
  const long long q = Wt / C, r = Wt % C;
  const long long X0 = q * bi + (r * bi + C - 1) / C, X1 = q * (bi + 1) + (r * (bi + 1) + C - 1) / C;
  if (X0 >= X1) return;  // the whole CTA, before any copy is issued

  // A test-sized wait limit (mobi_debug_set_wait_limit below 64) first waits
  // on a barrier that nothing completes, so the timeout path runs
  // deterministically; every warp runs it out, so every warp stops here.
  if (limit < 64 && !__all_sync(0xffffffffu, dec_wait(never, 0, limit, st, 0x2ff))) return;

  // The first tile starting at or after X0: problem p, chunk c, tile b (b may
  // be one past the chunk's last tile; the loop moves on to the next chunk).
  int p = 0;
#pragma unroll 1
  for (int j = 1; j < G; ++j)
    if (sp.pre[j] <= X0) p = j;
  int c, b;
  {
    const long long x = X0 - sp.pre[p];
    const int nch = grp.p[p].nch;
    const long long cc = x / sp.chunk[p];
    c = (int)(cc < nch - 1 ? cc : nch - 1);
    const long long rem = x - (long long)c * sp.chunk[p] - kDecSegCost;
    const int u = c < nch - 1 ? sp.u_full[p] : sp.u_last[p];
    b = rem <= 0 ? 0 : (int)((rem + u - 1) / u);
  }

  const uint64_t policy = l2_evict_first_policy();
  uint8_t* const codes_ring = sm + L::kCodes + (uint32_t)warp * D * kDecCodes;
  uint8_t* const sz_ring = sm + L::kSzs + (uint32_t)warp * D * kDecSz;
  float2* const scw = reinterpret_cast<float2*>(sm + L::kSc) + warp * kDecChunk * kDecRows;
  float2* const head_mine = reinterpret_cast<float2*>(sm + L::kHead) + warp * NB * 2 * 32;
  const float2* const head_next = head_mine + NB * 2 * 32;
  const float* const xs_sm = reinterpret_cast<const float*>(sm + L::kXs);
  const uint32_t bimg = smem_addr(sm + L::kBimg) + (uint32_t)lane * 16;

  // 2-bit codes: words 2 t4, 2 t4 + 1 of group g for row r of the tile: half
  // g / 4, 16-byte chunk 2 (g % 4) + t4 / 2 stored at chunk ^ (r % 8), rows
  // 128 bytes. 1-bit codes: word t4 of group g, 16-byte chunk g stored at
  // g ^ (r % 8); its even bits are the codes of 2-bit word 2 t4 and its odd
  // bits those of word 2 t4 + 1, so (w, w >> 1) take the place of that pair.
  // With per-slice widths (BITS 3) coff holds the 2-bit offsets and the 1-bit
  // ones are formed when needed.
  uint32_t coff[kDecChunk];
#pragma unroll
  for (int g = 0; g < kDecChunk; ++g)
    coff[g] = BITS != 1 ? (uint32_t)(g >> 2) * kDecHalf + (uint32_t)gid * 128u +
                              (uint32_t)((((g & 3) * 2 + (t4 >> 1)) ^ gid) * 16) + (t4 & 1) * 8u
                        : (uint32_t)gid * 128u + (uint32_t)((g ^ gid) * 16) + (uint32_t)t4 * 4u;

  bool ok = true;
  uint32_t issued = 0, done = 0;  // stages this warp has issued / consumed (ring slot = count % D)
  // A tile this warp left unfinished at the end of the previous segment (its
  // first slices, parked in the warp's scale/zero scratch); the next warp
  // holds the rest in its head slot.
  bool tail = false;

#pragma unroll 1
  for (;;) {
    // ---- the next segment: tiles b .. b_end - 1 of chunk c of problem p ----
    if (p < G && b >= grp.p[p].nblocks) {
      b = 0;
      if (++c == grp.p[p].nch) {
        c = 0;
        ++p;
      }
    }
    bool more = p < G;
    int km = 1, b_end = 0, a = 0, a1 = 0;
    // The chunk of X (for the B image) and k_t are loaded before this
    // segment's first stages are requested, so they return ahead of them.
    constexpr int kMaxVec = (8 * NB * kDecChunk * 16 + L::kThreads - 1) / L::kThreads;
    uint4 raw[kMaxVec];
    int my_kt = 0, g_valid = 0, nvec = 0;
    if (more) {
      const int nch = grp.p[p].nch, tiles = grp.p[p].nblocks;
      const int u = c < nch - 1 ? sp.u_full[p] : sp.u_last[p];
      const long long base = sp.pre[p] + (long long)c * sp.chunk[p] + kDecSegCost;  // start of tile 0
      more = base + (long long)b * u < X1;
      if (more) {
        km = sp.km[p];
        const long long be = (X1 - base + u - 1) / u;  // tiles starting before X1
        b_end = be < tiles ? (int)be : tiles;
        const int nt = b_end - b, ns = nt * km;
        if (ns >= kDecWarps * km) {  // even runs of stages, cut only before a tile's last slice
          a = dec_cut(warp * ns / kDecWarps, km);
          a1 = dec_cut((warp + 1) * ns / kDecWarps, km);
        } else {  // whole tiles, one per warp
          a = (warp < nt ? warp : nt) * km;
          a1 = (warp + 1 < nt ? warp + 1 : nt) * km;
        }
        const DecProblem& pr = grp.p[p];
        g_valid = pr.ngroups - c * kDecChunk < kDecChunk ? pr.ngroups - c * kDecChunk : kDecChunk;
        nvec = pr.T * g_valid * 16;  // 8-element vectors of X in this chunk
        my_kt = lane < pr.T ? pr.k_t[lane] : 0;
#pragma unroll
        for (int i = 0; i < kMaxVec; ++i) {
          const int v = threadIdx.x + i * L::kThreads;
          if (v < nvec) {
            const int t = v / (g_valid * 16), rr = v - t * (g_valid * 16);
            raw[i] = __ldg(reinterpret_cast<const uint4*>(pr.X + (int64_t)t * pr.K +
                                                          (int64_t)(c * kDecChunk + (rr >> 4)) * 128 + (rr & 15) * 8));
          }
        }
        // The first D - 1 stages go out before the segment's set-up.
        const int nramp = a1 - a < D - 1 ? a1 - a : D - 1;
        if (lane == 0 && ok) {
          for (int k = 0; k < nramp; ++k) {
            const uint32_t slot = (issued + k) % D;
            const int jj = a + k;
            const int tt = b + jj / km, ss = jj % km;
            const int bw = dec_width<BITS>(grp.mask1, ss);
            dec_issue(&grp.tm_codes[p][BITS == 3 ? ss : 0], &grp.tm_sz[p], codes_ring + slot * kDecCodes,
                      sz_ring + slot * kDecSz, &full[slot], (BITS == 3 ? 0 : ss * pr.N) + tt * kDecRows, bw, tt, ss,
                      pr.ngroups, c, policy);
          }
        }
        if (ok) issued += nramp;
      }
    }
    __syncthreads();  // every warp is done with the previous segment (image, head slots)
    ok = *reinterpret_cast<volatile int*>(&s_abort) == 0;
    if (tail) {  // finish the tile left by this warp: its slices so far plus the next warp's last slice
      if (ok) {
        float2 tA[NB], tB[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const float2 hA = head_next[(nb * 2 + 0) * 32 + lane], hB = head_next[(nb * 2 + 1) * 32 + lane];
          const float2 mA = scw[(nb * 2 + 0) * 32 + lane], mB = scw[(nb * 2 + 1) * 32 + lane];
          tA[nb] = make_float2(mA.x + hA.x, mA.y + hA.y);
          tB[nb] = make_float2(mB.x + hB.x, mB.y + hB.y);
        }
        dec_write_tile<NB>(s_tail_o[warp], s_tail_tn[warp].x, s_tail_tn[warp].y, gid, t4, tA, tB);
      }
      tail = false;
    }
    if (!more || !ok) break;

    const DecProblem& prob = grp.p[p];
    const int T = prob.T, N = prob.N, ngroups = prob.ngroups;

    // ---- the chunk's B image (zero beyond T tokens and beyond the last group) ----
    {
      uint4* img = reinterpret_cast<uint4*>(sm + L::kBimg);
      for (uint32_t i = threadIdx.x; i < L::kBimgBytes / 16; i += blockDim.x) img[i] = make_uint4(0u, 0u, 0u, 0u);
      __syncthreads();
      uint16_t* img16 = reinterpret_cast<uint16_t*>(sm + L::kBimg);
      bool bad = false;
#pragma unroll
      for (int i = 0; i < kMaxVec; ++i) {
        const int v = threadIdx.x + i * L::kThreads;
        if (v < nvec) {
          const int t = v / (g_valid * 16), rr = v - t * (g_valid * 16);
          const int g = rr >> 4, k0 = (rr & 15) * 8;  // k0 = 32 t4 + 16 m + 8 e
          const uint32_t uu[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
          const int tt4 = k0 >> 5, m = (k0 >> 4) & 1, e = (k0 >> 3) & 1;
          const int nb = t >> 3, n = t & 7, cc = 2 * tt4 + e;
#pragma unroll
          for (int qq = 0; qq < 8; ++qq) {  // element k0 + qq: h = qq >> 2, f = qq & 3
            const uint32_t bits = (uu[qq >> 1] >> (16 * (qq & 1))) & 0xffffu;
            bad |= (bits & 0x7F80u) >= (158u << 7);
            const int h = qq >> 2, f = qq & 3, j = 4 * h + f;
            const float v32 = __uint_as_float(bits << 16) * __uint_as_float((uint32_t)(127 + 96 - 2 * f) << 23);
            img16[(bimg_off(g, nb, j, m, NB) + (uint32_t)n * 16 + (uint32_t)cc * 2) >> 1] =
                (uint16_t)(__float_as_uint(v32) >> 16);  // exact: a power-of-two scaling of a bf16
          }
        }
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) report_error(st, kErrInputRange, 0x100);
      __syncthreads();
    }
    // ---- group sums on the tensor core: codes all 1 -> every D row is sum_k x * 2^-37 ----
    if (warp < kDecChunk) {
      const int g = warp;
      const uint32_t base = smem_addr(sm + L::kBimg);
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
        for (int jp = 0; jp < 4; ++jp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(base + bimg_off(g, nb, 2 * jp, 0, NB) + (uint32_t)lane * 16, b0, b1, b2, b3);
          const uint32_t one0 = 0x00010001u << (2 * ((2 * jp) & 3)), one1 = 0x00010001u << (2 * ((2 * jp + 1) & 3));
          mma_bf16_16816(d, one0, one0, one0, one0, b0, b1);
          mma_bf16_16816(d, one1, one1, one1, one1, b2, b3);
        }
        if (gid == 0) {
          float* xs = reinterpret_cast<float*>(sm + L::kXs) + g * 16 + 8 * nb + 2 * t4;
          xs[0] = d[0] * kTwo37;
          xs[1] = d[1] * kTwo37;
        }
      }
    }
    __syncthreads();

    float2 yA[NB], yB[NB];  // rows gid (A) and gid + 8 (B), tokens 8 nb + 2 t4 + {0, 1}
    // k_t of the tokens whose columns this lane holds: 8 nb + 2 t4 + e.
    int ktl[NB][2];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
      ktl[nb][0] = __shfl_sync(0xffffffffu, my_kt, 8 * nb + 2 * t4);
      ktl[nb][1] = __shfl_sync(0xffffffffu, my_kt, 8 * nb + 2 * t4 + 1);
    }
    // sum_k x of the lane's two tokens, per group and column block.
    constexpr bool kJitB = DecCfg<NB>::kJitB, kXsSmem = DecCfg<NB>::kXsSmem;
    float2 xs[kXsSmem ? 1 : kDecChunk][NB];
    if constexpr (!kXsSmem) {
#pragma unroll
      for (int g = 0; g < kDecChunk; ++g)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb)
          xs[g][nb] = *reinterpret_cast<const float2*>(xs_sm + g * 16 + 8 * nb + 2 * t4);
    }

    float* const out = prob.out + (int64_t)c * T * N;
    const CUtensorMap* tm_sz = &grp.tm_sz[p];
    int s = a % km, tile = b + a / km;  // consumer cursor
    bool head = s != 0;                 // the first tile's other slices are the previous warp's
    int pj = a + (a1 - a < D - 1 ? a1 - a : D - 1);
    int ps = pj % km, ptile = b + pj / km;  // producer cursor
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) yA[nb] = yB[nb] = make_float2(0.0f, 0.0f);

#pragma unroll 1
    for (int j = a; j < a1; ++j) {
      const uint32_t slot = done % D;
      // Refill the slot read in the previous iteration (every lane is done with it).
      __syncwarp();
      if (pj < a1) {
        const uint32_t ns = issued % D;
        if (lane == 0)
          dec_issue(&grp.tm_codes[p][BITS == 3 ? ps : 0], tm_sz, codes_ring + ns * kDecCodes,
                    sz_ring + ns * kDecSz, &full[ns], (BITS == 3 ? 0 : ps * N) + ptile * kDecRows,
                    dec_width<BITS>(grp.mask1, ps), ptile, ps, ngroups, c, policy);
        ++issued;
        ++pj;
        if (++ps == km) {
          ps = 0;
          ++ptile;
        }
      }
      if (!(ok = __all_sync(0xffffffffu, dec_wait(&full[slot], (done / D) & 1u, limit, st, 0x200 + s)))) {
        if (lane == 0) *reinterpret_cast<volatile int*>(&s_abort) = 1;
        break;
      }
      ++done;
      const uint8_t* cs = codes_ring + slot * kDecCodes;
      const bool w1 = dec_width<BITS>(grp.mask1, s) == 1;  // this stage's codes are 1-bit
      const uint32_t field_mask = w1 ? 0x00010001u : 0x00030003u;
      // Scale/zero words of the stage as fp32 pairs (scale 2^37, -scale zero),
      // one conversion per word for the whole warp.
      {
        const uint32_t* szw = reinterpret_cast<const uint32_t*>(sz_ring + slot * kDecSz);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t w = szw[lane + 32 * i];
          const float sc = __half2float(__ushort_as_half((unsigned short)(w & 0xffffu)));
          const float zf = __half2float(__ushort_as_half((unsigned short)(w >> 16)));
          scw[lane + 32 * i] = make_float2(sc * kTwo37, -sc * zf);
        }
        __syncwarp();
      }
      float2 ysA[NB], ysB[NB];
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) ysA[nb] = ysB[nb] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int g0 = 0; g0 < kDecChunk; g0 += 2) {
        if (g0 >= g_valid) break;  // the last chunk's missing groups (their B image is zero)
        uint2 wa[2], wb[2];
        // B fragments: all eight k16 steps of both groups up front, or (kJitB)
        // two steps at a time just before their MMAs.
        uint32_t bf[2][NB][kJitB ? 2 : 8][2];
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          if (!w1) {
            wa[gg] = *reinterpret_cast<const uint2*>(cs + coff[g0 + gg]);
            wb[gg] = *reinterpret_cast<const uint2*>(cs + coff[g0 + gg] + 8 * 128);
          } else {
            const uint32_t o1 = BITS == 1 ? coff[g0 + gg]
                                          : (uint32_t)gid * 128u + (uint32_t)(((g0 + gg) ^ gid) * 16) + (uint32_t)t4 * 4u;
            const uint32_t x = *reinterpret_cast<const uint32_t*>(cs + o1);
            const uint32_t y = *reinterpret_cast<const uint32_t*>(cs + o1 + 8 * 128);
            wa[gg] = make_uint2(x, x >> 1);
            wb[gg] = make_uint2(y, y >> 1);
          }
          if constexpr (!kJitB) {
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
              for (int jp = 0; jp < 4; ++jp)
                ldsm_x4(bimg + bimg_off(g0 + gg, nb, 2 * jp, 0, NB), bf[gg][nb][2 * jp][0], bf[gg][nb][2 * jp][1],
                        bf[gg][nb][2 * jp + 1][0], bf[gg][nb][2 * jp + 1][1]);
          }
        }
        float d[2][NB][4];
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int h = jj >> 2, f = jj & 3;
          const uint32_t mk = field_mask << (2 * f);
          const int jb = kJitB ? (jj & 1) : jj;  // the step's slot in bf
          if constexpr (kJitB) {
            if ((jj & 1) == 0) {
#pragma unroll
              for (int gg = 0; gg < 2; ++gg)
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
                  ldsm_x4(bimg + bimg_off(g0 + gg, nb, jj, 0, NB), bf[gg][nb][0][0], bf[gg][nb][0][1],
                          bf[gg][nb][1][0], bf[gg][nb][1][1]);
            }
          }
#pragma unroll
          for (int gg = 0; gg < 2; ++gg) {
            const uint32_t a0 = (wa[gg].x >> (8 * h)) & mk, a2 = (wa[gg].y >> (8 * h)) & mk;
            const uint32_t a1r = (wb[gg].x >> (8 * h)) & mk, a3 = (wb[gg].y >> (8 * h)) & mk;
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
              if (jj == 0) mma_bf16_16816_z(d[gg][nb], a0, a1r, a2, a3, bf[gg][nb][jb][0], bf[gg][nb][jb][1]);
              else mma_bf16_16816(d[gg][nb], a0, a1r, a2, a3, bf[gg][nb][jb][0], bf[gg][nb][jb][1]);
            }
          }
        }
        // Per-group promotion: ys += scale 2^37 acc - scale z sum_k x.
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
          const int g = g0 + gg;
          const float2 pA = scw[g * kDecRows + gid], pB = scw[g * kDecRows + gid + 8];
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const float2 xg =
                kXsSmem ? *reinterpret_cast<const float2*>(xs_sm + g * 16 + 8 * nb + 2 * t4) : xs[kXsSmem ? 0 : g][nb];
            ysA[nb] = __ffma2_rn(make_float2(pA.x, pA.x), make_float2(d[gg][nb][0], d[gg][nb][1]),
                                 __ffma2_rn(make_float2(pA.y, pA.y), xg, ysA[nb]));
            ysB[nb] = __ffma2_rn(make_float2(pB.x, pB.x), make_float2(d[gg][nb][2], d[gg][nb][3]),
                                 __ffma2_rn(make_float2(pB.y, pB.y), xg, ysB[nb]));
          }
        }
      }
      // The slice counts only for the tokens that take it (k_t > s).
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        const float2 m = make_float2(ktl[nb][0] > s ? 1.0f : 0.0f, ktl[nb][1] > s ? 1.0f : 0.0f);
        yA[nb] = __ffma2_rn(m, ysA[nb], yA[nb]);
        yB[nb] = __ffma2_rn(m, ysB[nb], yB[nb]);
      }
      if (++s == km) {
        if (head) {  // the last slice of a tile the previous warp started: it adds this after the barrier
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            head_mine[(nb * 2 + 0) * 32 + lane] = yA[nb];
            head_mine[(nb * 2 + 1) * 32 + lane] = yB[nb];
          }
          head = false;
        } else {
          dec_write_tile<NB>(out + tile * kDecRows, T, N, gid, t4, yA, yB);
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) yA[nb] = yB[nb] = make_float2(0.0f, 0.0f);
        s = 0;
        ++tile;
      }
    }
    if (ok && s != 0) {  // this warp's run ended inside a tile: finished after the next barrier
      tail = true;
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) {
        scw[(nb * 2 + 0) * 32 + lane] = yA[nb];
        scw[(nb * 2 + 1) * 32 + lane] = yB[nb];
      }
      if (lane == 0) {
        s_tail_o[warp] = out + tile * kDecRows;
        s_tail_tn[warp] = make_int2(T, N);
      }
    }
    b = b_end;
  }
  // Every copy this warp issued lands before the CTA may exit: normally all
  // have been waited for; after a timeout the stages still in flight are
  // drained here.
  __syncwarp();
  if (lane == 0)
    for (uint32_t i = done; i < issued; ++i) mbar_wait(&full[i % D], (i / D) & 1u, kDefaultWaitLimit, st, 0x2f0);
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

template <int NB, int MG, int BITS>
static cudaError_t launch_decode_class(const DecGroup<MG, BITS>& grp, int ctas, cudaStream_t stream,
                                       DeviceStatus* st) {
  using L = DecLayout<NB>;
  cudaError_t e = set_smem((const void*)decode_kernel<NB, MG, BITS>, (int)L::kDynamic);
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
  e = cudaLaunchKernelEx(&cfg, decode_kernel<NB, MG, BITS>, grp, st, wait_limit());
  if (e != cudaSuccess) return note_error("decode launch", e);
  return note_error("kernel launch", cudaGetLastError());
}

// Fills a table of capacity MG with the problems `idx[0..n)` of one fragment
// class and launches it on one CTA per SM; the kernel itself shares the CTAs
// among the problems once it knows their k_t. Problems with several chunks are
// appended to `red`.
template <int MG, int BITS>
static cudaError_t decode_class(const DecodeJob* jobs, const int* idx, int n, int cls, int S, int sms,
                                DecReduceGroup* red, cudaStream_t stream, DeviceStatus* st) {
  DecGroup<MG, BITS> grp;
  memset(&grp, 0, sizeof grp);
  grp.G = n;
  grp.S = S;
  grp.mask1 = n > 0 ? jobs[idx[0]].mask1 : 0;
  for (int m = 0; m < n; ++m) {
    const DecodeJob& j = jobs[idx[m]];
    const int64_t nch = dec_chunks(j.K), nblocks = (j.N + kDecRows - 1) / kDecRows;
    if (BITS != 3) {
      const uint64_t words = (uint64_t)(j.K / 32 * BITS);  // per row and slice
      if (!make_tmap_2d(&grp.tm_codes[m][0], j.codes, 4, words, (uint64_t)(S * j.N), words * 4, 32, kDecRows, 128))
        return note_error("decode tensor map (codes)", cudaErrorInvalidValue);
    } else {  // one map per slice: slice s starts after the words of slices 0 .. s-1
      const uint32_t* base = j.codes;
      for (int sl = 0; sl < S; ++sl) {
        const int w = ((j.mask1 >> sl) & 1) ? 1 : 2;
        const uint64_t words = (uint64_t)(j.K / 32 * w);
        if (!make_tmap_2d(&grp.tm_codes[m][sl], base, 4, words, (uint64_t)j.N, words * 4, 32, kDecRows, 128))
          return note_error("decode tensor map (codes of a slice)", cudaErrorInvalidValue);
        base += (size_t)j.N * words;
      }
    }
    if (!make_tmap_2d(&grp.tm_sz[m], j.sz, 4, (uint64_t)j.N, (uint64_t)(S * (j.K / 128)), (uint64_t)j.N * 4,
                      kDecRows, kDecChunk, 0))
      return note_error("decode tensor map (scale/zero)", cudaErrorInvalidValue);
    grp.p[m] = DecProblem{static_cast<const __nv_bfloat16*>(j.X), j.k_t, nch > 1 ? j.partial : j.Y, j.T, (int)j.N,
                          (int)j.K, (int)(j.K / 128), (int)nblocks, (int)nch};
    if (nch > 1) {
      red->partial[red->G] = reinterpret_cast<const float4*>(j.partial);
      red->Y[red->G] = reinterpret_cast<float4*>(j.Y);
      red->nch[red->G] = (int)nch;
      red->off[red->G + 1] = red->off[red->G] + (int64_t)j.T * j.N / 4;
      ++red->G;
    }
  }
  return cls == 1 ? launch_decode_class<1, MG, BITS>(grp, sms, stream, st)
                  : launch_decode_class<2, MG, BITS>(grp, sms, stream, st);
}

// One launch per fragment class present (T <= 8, then 9 <= T <= 16), each a
// persistent grid of one CTA per SM that the kernel shares among that class's
// problems in equal parts of the slices they read, then one chunk-reduction launch for
// every problem with more than one chunk. Each launch is a programmatic
// dependent of the one before (the decode kernel reads k_t, which decides its
// work split, only after the kernel before has finished).
cudaError_t launch_decode_grouped(const DecodeJob* jobs, int G, int S, cudaStream_t stream, DeviceStatus* st) {
  const int sms = num_sms();
  DecReduceGroup red = {};
  red.off[0] = 0;
  for (int cls = 1; cls <= 2; ++cls)
    for (int bits = 3; bits >= 1; --bits) {
      int idx[kMaxGroup];
      int n = 0;
      for (int i = 0; i < G; ++i) {
        const DecodeJob& j = jobs[i];
        if (j.T > 0 && j.N > 0 && (j.T > 8 ? 2 : 1) == cls && j.bits == bits) idx[n++] = i;
      }
      if (n == 0) continue;
      cudaError_t e;
      if (bits == 2)
        e = n == 1 ? decode_class<1, 2>(jobs, idx, n, cls, S, sms, &red, stream, st)
                   : decode_class<kMaxGroup, 2>(jobs, idx, n, cls, S, sms, &red, stream, st);
      else if (bits == 1)
        e = n == 1 ? decode_class<1, 1>(jobs, idx, n, cls, S, sms, &red, stream, st)
                   : decode_class<kMaxGroup, 1>(jobs, idx, n, cls, S, sms, &red, stream, st);
      else
        e = n == 1 ? decode_class<1, 3>(jobs, idx, n, cls, S, sms, &red, stream, st)
                   : decode_class<kMaxGroup, 3>(jobs, idx, n, cls, S, sms, &red, stream, st);
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
                          DeviceStatus* st, int bits, int mask1) {
  const DecodeJob job{X, k_t, codes, sz, Y, static_cast<float*>(ws), N, K, T, bits, mask1};
  return launch_decode_grouped(&job, 1, S, stream, st);
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
      launch_decode(X, (int)T, K, k_t, codes, sz, N, S, Y, scratch, static_cast<cudaStream_t>(stream), st, 2,
                    0));
}
