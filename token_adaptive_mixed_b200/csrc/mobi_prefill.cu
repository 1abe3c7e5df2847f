// mobi_prefill.cu — prefill GEMM (any T, used for T > 16) of the token-routed
// mixed-bit linear layer on sm_100a: tcgen05 tensor cores, TMEM accumulators,
// TMA-staged tiles.
//
// y[t,n] = sum_{s < k_t} sum_g scale[s,g,n] * sum_{k in g} x[t,k] (q[s,n,k] - z[s,g,n])
// (MoBiQuant explainer [ja] §2.1 W^(b) = sum W_e; [en] §2.A "Elasticity"),
// fp32 accumulation, exact operands.
//
// Tokens are taken in bucket order (perm from the routing step, ascending
// k_t). A tile is 128 weight rows x 192 consecutive bucket-ordered tokens; for
// group g and slice s < kmax(tile) one "unit" computes
//   D[n, t] = sum_{k in g} (q - z)[s, n, k] * x[t, k]
// with 8 tcgen05.mma (M=128, N=192, K=16, bf16 in, fp32 in TMEM), and the
// epilogue promotes acc[n, t] += scale[s,g,n] * D[n, t] for the tokens that take
// slice s (a suffix of the tile's columns, since tokens are sorted by k_t).
//
// Operands:
//   A (weights) lives in tensor memory: four dequant warps turn the 2-bit codes
//     of their rows into exact bf16 (q - z) pairs and write them with
//     tcgen05.st, so the dequantised operand never touches shared memory.
//     With w the packed word, ((w >> sh) & (0x00030003 << 2f)) | 0x43004300 is
//     the bf16 pair (128 + 4^f q); one bf16x2 FMA by 4^-f minus (128 / 4^f + z)
//     gives q - z exactly, so each pair costs one logic op and one FMA (plus a
//     shift shared by three pairs). A 1-bit word w (32 codes) is read as the
//     2-bit-field pair (w, w >> 1) with the masks 0x00010001 << 2f: its even
//     bits are the codes of one 16-code block, its odd bits the next. Each
//     slice may have its own width (one code map per slice).
//   B (tokens) comes from shared memory: one bulk copy per group brings a
//     192-token x tile that the gather kernel has already laid out as the
//     128-byte-swizzled shared-memory image (rows in bucket order and, within
//     each 16-column block, columns interleaved as (c, c+8) to match the pair
//     order of the packed words).
// Pipeline: units flow through two accumulator buffers in TMEM (D, 2 x 192
// columns) and the A operand through four half-group slots (4 x 32 columns), so
// the MMA of a unit overlaps both the epilogue of the one before and the
// dequantisation of the next; the MMA can start on the first half of a group
// while its second half is still being dequantised.
// Warp roles (16 warps): 0 TMA producer, 1 and 2 MMA issuers (even and odd
// units; warp 1 also owns TMEM), 4-7 dequant (one per TMEM lane quadrant),
// 8-15 epilogue (two per quadrant, 96 token columns each); warp 3 only takes
// part in set-up and teardown.
// All mbarrier waits are bounded; on a timeout the kernel records the error,
// stops issuing, drains its copies and MMAs in flight, frees TMEM and returns.
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "mobi_device.cuh"
#include "mobi_host.h"

namespace mobi {

namespace pf {
constexpr int BM = 128;          // weight rows per tile (tcgen05 M)
constexpr int XST = 3;           // x-tile stages (one group each)
constexpr int CST = 6;           // code/scale stages (one unit each)
constexpr int DST = 2;           // accumulator buffers in TMEM (one unit each)
constexpr int AST = 4;           // A-operand slots in TMEM (one half group each)
// 16 warps launched with 128 registers each; the warpgroups then rebalance
// registers (setmaxnreg): producer/MMA 40, dequant 80, epilogue 168.
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kDeqWarp0 = 4;
constexpr int kEpiWarp0 = 8;
constexpr int kEpiWarps = 8;                   // two per TMEM lane quadrant
constexpr uint32_t kCodeBytes = BM * 32;       // 128 rows x 8 words (2-bit codes; 4 words for 1-bit)
constexpr uint32_t kSzBytes = BM * 4;
constexpr uint32_t kTmemCols = 512;

// Token-tile width BN (tcgen05 N): 192 for prefill, 64 for small batches
// (up to 64 tokens, where a 192-wide tile would be mostly padding).
template <int BN_>
struct Tile {
  static constexpr int BN = BN_;
  static constexpr int kColsPerEpi = BN / 2;                // token columns per epilogue warp
  static constexpr int kChunkCols = BN == 192 ? 48 : 32;    // columns per TMEM wait in the epilogue
  static constexpr uint32_t kXHalfBytes = BN * 128;         // BN rows x 64 bf16
  static constexpr uint32_t kXStageBytes = 2 * kXHalfBytes;
  static constexpr uint32_t kTmemD = 0;                     // D slot j at columns j * BN
  static constexpr uint32_t kTmemA = DST * BN;              // A slot j at columns kTmemA + 32 j
  static_assert(DST * BN + AST * 32 <= (int)kTmemCols, "TMEM budget");
  static_assert(kColsPerEpi % kChunkCols == 0 && kChunkCols % 16 == 0, "epilogue chunks");
};
}  // namespace pf

// Code maps of the packed slices: one map over every slice (per_slice 0, row
// s N + n) or one per slice (per_slice 1, row n); slice s has 1-bit codes when
// bit s of mask1 is set, 2-bit codes otherwise.
struct PfCodeMaps {
  CUtensorMap m[kMaxSlices];
  int per_slice;
  int mask1;
};

template <int BN>
struct PfSmem {
  uint8_t x[pf::XST][pf::Tile<BN>::kXStageBytes];     // 1024-byte aligned (offset 0)
  uint32_t codes[pf::CST][pf::BM * 8];      // [row][word]
  uint32_t sz[pf::CST][pf::BM];
  uint64_t x_full[pf::XST], x_empty[pf::XST];
  uint64_t c_full[pf::CST], c_empty[pf::CST];
  uint64_t a_full[pf::AST], a_empty[pf::AST];
  uint64_t d_full[pf::DST], d_empty[pf::DST];
  uint64_t drain;
  uint32_t tmem_base;
  int32_t abort_flag;
};

// ---- tile bookkeeping ------------------------------------------------------------------

struct TileInfo {
  int64_t n0;      // first weight row
  int64_t t0;      // first bucket-ordered token
  int64_t g0, g1;  // the tile's groups [g0, g1) along K
  int kc;          // its K chunk
  int nvalid;      // tokens in the tile
  int kmax;        // slices needed by the tile (k of its last token)
  int lo[kMaxSlices];  // first tile column whose token takes slice s
};

// Tile index = (weight tile * n_tt + token tile) * nkc + K chunk; a chunk is
// gpc consecutive groups.
template <int BN, bool KSPLIT>
__device__ __forceinline__ TileInfo tile_info(int64_t tile, int64_t n_tt, int nkc, int64_t gpc, int64_t ngroups,
                                              int64_t T, const int32_t* off, int S) {
  TileInfo ti;
  if constexpr (!KSPLIT) {  // one K chunk: the whole K
    nkc = 1;
    gpc = ngroups;
  }
  const int64_t kc = tile % nkc, rest = tile / nkc;
  const int64_t wt = rest / n_tt, tt = rest % n_tt;
  ti.kc = (int)kc;
  ti.g0 = kc * gpc;
  ti.g1 = ti.g0 + gpc < ngroups ? ti.g0 + gpc : ngroups;
  ti.n0 = wt * pf::BM;
  ti.t0 = tt * BN;
  ti.nvalid = (int)(T - ti.t0 < BN ? T - ti.t0 : BN);
  const int64_t last = ti.t0 + ti.nvalid - 1;
  int km = 1;
#pragma unroll
  for (int j = 1; j < kMaxSlices; ++j)
    if (j < S && (int64_t)off[j] <= last) km = j + 1;
  ti.kmax = km;
#pragma unroll
  for (int s = 0; s < kMaxSlices; ++s) {
    int64_t l = s < S ? (int64_t)off[s] - ti.t0 : 0;
    l = l < 0 ? 0 : (l > ti.nvalid ? ti.nvalid : l);
    ti.lo[s] = (int)l;
  }
  return ti;
}

// The i-th tile of this CTA, or -1 past the last. Tiles are dealt largest
// first: token tiles in descending order (in bucket order a later token tile
// needs as many slices or more) and, within one, the weight tiles in order;
// pass i deals one tile to every CTA, in CTA order on even passes and in
// reverse on odd ones, so heavy and light tiles even out across CTAs.
__device__ __forceinline__ int64_t pf_tile(int64_t i, int64_t ntiles, int64_t n_wt, int64_t n_tt, int nkc) {
  const int64_t G = gridDim.x, c = blockIdx.x;
  const int64_t idx = i * G + ((i & 1) ? G - 1 - c : c);
  if (idx >= ntiles) return -1;
  const int64_t per_tt = n_wt * nkc;
  const int64_t tt = n_tt - 1 - idx / per_tt, r = idx % per_tt;
  const int64_t wt = r / nkc, kc = r % nkc;
  return (wt * n_tt + tt) * nkc + kc;
}

// Bounded wait that also gives up when another role has aborted.
__device__ __forceinline__ bool pf_wait(uint64_t* bar, uint32_t parity, uint64_t limit, DeviceStatus* st,
                                        uint32_t where, volatile int32_t* abort_flag) {
  for (uint64_t i = 0; i < limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 255 && *abort_flag) return false;
  }
  report_error(st, kErrTimeout, where);
  *abort_flag = 1;
  return false;
}

// Y: the output [T][N] when nkc == 1, else the per-chunk partials [nkc][T][N]
// (added in chunk order by a separate reduction). KSPLIT = false compiles the
// single-chunk kernel (nkc ignored), which keeps the K-chunk bookkeeping out
// of its registers.
template <int BN, bool KSPLIT>
__global__ void __launch_bounds__(pf::kThreads, 1) prefill_kernel(
    const uint8_t* __restrict__ Xt, const __grid_constant__ PfCodeMaps tm_codes,
    const __grid_constant__ CUtensorMap tm_sz, const uint32_t* __restrict__ sz, const int32_t* __restrict__ perm,
    const int32_t* __restrict__ offsets, int64_t T, int64_t N, int64_t ngroups, int S, int nkc,
    float* __restrict__ Y, DeviceStatus* st, uint64_t limit) {
  using TL = pf::Tile<BN>;
  if constexpr (!KSPLIT) nkc = 1;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // Dynamic shared memory is rounded up to a 1024-byte boundary for the swizzled tiles.
  PfSmem<BN>& sm = *reinterpret_cast<PfSmem<BN>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int32_t* abort_flag = &sm.abort_flag;
  (void)sz;

  const int64_t n_wt = (N + pf::BM - 1) / pf::BM;
  const int64_t n_tt = (T + BN - 1) / BN;
  const int64_t ntiles = n_wt * n_tt * nkc;
  const int64_t gpc = (ngroups + nkc - 1) / nkc;  // groups per K chunk
  int32_t off[kMaxSlices + 1];
#pragma unroll
  for (int j = 0; j <= kMaxSlices; ++j) off[j] = j <= S ? __ldg(offsets + j) : 0;

  if (threadIdx.x == 0) {
    // An x stage is released by both MMA issuers (each commits after its own MMAs).
    for (int i = 0; i < pf::XST; ++i) { mbar_init(&sm.x_full[i], 1); mbar_init(&sm.x_empty[i], 2); }
    // A code/scale stage is released by the 4 dequant warps and the 8 epilogue
    // warps (which read the scales from it).
    for (int i = 0; i < pf::CST; ++i) { mbar_init(&sm.c_full[i], 1); mbar_init(&sm.c_empty[i], 4 + pf::kEpiWarps); }
    for (int i = 0; i < pf::AST; ++i) { mbar_init(&sm.a_full[i], 4); mbar_init(&sm.a_empty[i], 1); }
    for (int i = 0; i < pf::DST; ++i) { mbar_init(&sm.d_full[i], 1); mbar_init(&sm.d_empty[i], pf::kEpiWarps); }
    mbar_init(&sm.drain, 2);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(&sm.tmem_base, pf::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Each warpgroup rebalances its registers (setmaxnreg) at the top of its role.
  if (warp < 4) {
   asm volatile("setmaxnreg.dec.sync.aligned.u32 40;");
   if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      for (int j = 0; j < (tm_codes.per_slice ? S : 1); ++j) prefetch_tmap(&tm_codes.m[j]);
      prefetch_tmap(&tm_sz);
      uint32_t xi = 0, ci = 0;  // running stage counters
      bool ok = true;
      for (int64_t i = 0, tile; (tile = pf_tile(i, ntiles, n_wt, n_tt, nkc)) >= 0 && ok; ++i) {
        const TileInfo ti = tile_info<BN, KSPLIT>(tile, n_tt, nkc, gpc, ngroups, T, off, S);
        for (int64_t g = ti.g0; g < ti.g1 && ok; ++g) {
          const uint32_t xs = xi % pf::XST, xph = (xi / pf::XST) & 1;
          if (!(ok = pf_wait(&sm.x_empty[xs], xph ^ 1, limit, st, 0x301, abort_flag))) break;
          mbar_arrive_expect_tx(&sm.x_full[xs], TL::kXStageBytes);
          // Pre-swizzled tile (token tile, group g): one contiguous bulk copy.
          const int64_t tt = ti.t0 / BN;
          bulk_g2s(&sm.x[xs][0], Xt + (tt * ngroups + g) * (int64_t)TL::kXStageBytes, TL::kXStageBytes,
                   &sm.x_full[xs]);
          ++xi;
          for (int s = 0; s < ti.kmax; ++s) {
            const uint32_t cs = ci % pf::CST, cph = (ci / pf::CST) & 1;
            if (!(ok = pf_wait(&sm.c_empty[cs], cph ^ 1, limit, st, 0x302, abort_flag))) break;
            const int bits = ((tm_codes.mask1 >> s) & 1) ? 1 : 2;
            mbar_arrive_expect_tx(&sm.c_full[cs], pf::kCodeBytes / 2 * bits + pf::kSzBytes);
            tma_load_2d(&sm.codes[cs][0], &tm_codes.m[tm_codes.per_slice ? s : 0], (int)(g * 4 * bits),
                        (int)((tm_codes.per_slice ? 0 : s * N) + ti.n0), &sm.c_full[cs]);
            tma_load_2d(&sm.sz[cs][0], &tm_sz, (int)ti.n0, (int)(s * ngroups + g), &sm.c_full[cs]);
            ++ci;
          }
        }
      }
      // Drain: every copy issued lands before the CTA may exit.
      for (uint32_t i = (xi > pf::XST ? xi - pf::XST : 0); i < xi; ++i)
        mbar_wait(&sm.x_full[i % pf::XST], (i / pf::XST) & 1, kDefaultWaitLimit, st, 0x3F1);
      for (uint32_t i = (ci > pf::CST ? ci - pf::CST : 0); i < ci; ++i)
        mbar_wait(&sm.c_full[i % pf::CST], (i / pf::CST) & 1, kDefaultWaitLimit, st, 0x3F2);
    }
   } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers ----------------
    // Two issuing threads in separate warps: warp 1 takes the even units and
    // owns D buffer 0 and A half-slots 0-1, warp 2 the odd units with D buffer 1
    // and A slots 2-3. A barrier check costs a few hundred cycles, so while one
    // thread checks the prerequisites of its next unit the other keeps the
    // tensor pipe fed. tcgen05.commit tracks the issuing thread's own MMAs, so
    // both threads release every x stage (count 2).
    if (lane == 0) {
      const uint32_t par = (uint32_t)(warp - 1);
      const uint32_t idesc = idesc_bf16(pf::BM, BN);
      uint32_t xi = 0, u = 0;  // x stages, units (all units are counted by both threads)
      bool ok = true;
      for (int64_t i = 0, tile; (tile = pf_tile(i, ntiles, n_wt, n_tt, nkc)) >= 0 && ok; ++i) {
        const TileInfo ti = tile_info<BN, KSPLIT>(tile, n_tt, nkc, gpc, ngroups, T, off, S);
        for (int64_t g = ti.g0; g < ti.g1 && ok; ++g) {
          const uint32_t xs = xi % pf::XST, xph = (xi / pf::XST) & 1;
          const uint32_t xbase = smem_addr(&sm.x[xs][0]);
          bool have_x = false;
          for (int s = 0; s < ti.kmax && ok; ++s, ++u) {
            if ((u & 1) != par) continue;
            if (!have_x) {
              if (!(ok = pf_wait(&sm.x_full[xs], xph, limit, st, 0x311, abort_flag))) break;
              have_x = true;
            }
            const uint32_t db = par, dph = (u >> 1) & 1;  // this thread's D buffer, its (u/2)-th use
            if (!(ok = pf_wait(&sm.d_empty[db], dph ^ 1, limit, st, 0x313, abort_flag))) break;
            // The dequant warps fill half 0 before half 1, so half 1 being full
            // covers both halves.
            const uint32_t hh1 = 2 * u + 1;
            if (!(ok = pf_wait(&sm.a_full[hh1 % pf::AST], (hh1 / pf::AST) & 1, limit, st, 0x312, abort_flag))) break;
            tc_fence_after();
            const uint32_t d_tmem = tmem + TL::kTmemD + db * BN;
            for (int half = 0; half < 2; ++half) {
              const uint32_t ab = (2 * u + half) % pf::AST;
              const uint32_t a_tmem = tmem + TL::kTmemA + ab * 32;
#pragma unroll
              for (int i = 0; i < 4; ++i) {  // k16 steps 4*half .. 4*half+3: one x half tile
                const uint32_t saddr = xbase + half * TL::kXHalfBytes + i * 32;
                mma_ts(d_tmem, a_tmem + 8 * i, desc_sw128(saddr), idesc, (half > 0 || i > 0) ? 1u : 0u);
              }
              mma_commit(&sm.a_empty[ab]);
            }
            mma_commit(&sm.d_full[db]);
          }
          if (!ok) break;
          mma_commit(&sm.x_empty[xs]);
          ++xi;
        }
      }
      // Drain: wait for every MMA issued so far before TMEM is released.
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, kDefaultWaitLimit, st, 0x3F3);
    }
   }
  } else if (warp >= pf::kDeqWarp0 && warp < pf::kDeqWarp0 + 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 80;");
    // ---------------- dequant: codes -> exact (q - z) bf16 pairs in TMEM ----------------
    const int q = warp & 3;               // TMEM lane quadrant of this warp
    const int r = 32 * q + lane;          // row within the tile
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    uint32_t u = 0, hh = 0;
    bool ok = true;
    for (int64_t i = 0, tile; (tile = pf_tile(i, ntiles, n_wt, n_tt, nkc)) >= 0 && ok; ++i) {
      const TileInfo ti = tile_info<BN, KSPLIT>(tile, n_tt, nkc, gpc, ngroups, T, off, S);
      for (int64_t g = ti.g0; g < ti.g1 && ok; ++g) {
        for (int s = 0; s < ti.kmax && ok; ++s, ++u) {
          const uint32_t cs = u % pf::CST, cph = (u / pf::CST) & 1;
          if (!(ok = pf_wait(&sm.c_full[cs], cph, limit, st, 0x321, abort_flag))) break;
          // The group's 128 codes of row r as eight 2-bit-field words: 2-bit
          // codes as stored; 1-bit codes (4 words) as (w, w >> 1) pairs, whose
          // even bits are the codes of the 2-bit words 2i and 2i + 1.
          const int bits = ((tm_codes.mask1 >> s) & 1) ? 1 : 2;
          uint32_t words[8];
          if (bits == 2) {
            const uint4 w0 = *reinterpret_cast<const uint4*>(&sm.codes[cs][r * 8]);
            const uint4 w1 = *reinterpret_cast<const uint4*>(&sm.codes[cs][r * 8 + 4]);
            words[0] = w0.x; words[1] = w0.y; words[2] = w0.z; words[3] = w0.w;
            words[4] = w1.x; words[5] = w1.y; words[6] = w1.z; words[7] = w1.w;
          } else {
            const uint4 w0 = *reinterpret_cast<const uint4*>(&sm.codes[cs][r * 4]);
            words[0] = w0.x; words[1] = w0.x >> 1; words[2] = w0.y; words[3] = w0.y >> 1;
            words[4] = w0.z; words[5] = w0.z >> 1; words[6] = w0.w; words[7] = w0.w >> 1;
          }
          const uint32_t fmask = bits == 2 ? 0x00030003u : 0x00010001u;
          const uint32_t zsz = sm.sz[cs][r];
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.c_empty[cs]);
          // FMA constants: v * 4^-f - (128 / 4^f + z) = q - z for the field at bit 2f.
          const float zf = __half2float(__ushort_as_half((unsigned short)(zsz >> 16)));
          __nv_bfloat162 mul[3], add[3];
#pragma unroll
          for (int f = 0; f < 3; ++f) {
            const float m = 1.0f / (float)(1 << (2 * f));
            mul[f] = __floats2bfloat162_rn(m, m);
            const float a = -(128.0f * m + zf);  // exact in bf16: 128 + z, 32 + z or 8 + z
            add[f] = __floats2bfloat162_rn(a, a);
          }
          // Both halves' slots first, then both halves stored, one store wait and
          // both arrivals (the MMA issuer waits for the second half only).
          const uint32_t ab0 = hh % pf::AST, ab1 = (hh + 1) % pf::AST;
          if (!(ok = pf_wait(&sm.a_empty[ab0], ((hh / pf::AST) & 1) ^ 1, limit, st, 0x322, abort_flag))) break;
          if (!(ok = pf_wait(&sm.a_empty[ab1], (((hh + 1) / pf::AST) & 1) ^ 1, limit, st, 0x322, abort_flag))) break;
          tc_fence_after();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const uint32_t ab = half ? ab1 : ab0;
            const uint32_t a_tmem = tmem + lane_addr + TL::kTmemA + ab * 32;
#pragma unroll
            for (int wp = 0; wp < 2; ++wp) {  // 16 columns (two words) per store
              uint32_t regs[16];
#pragma unroll
              for (int ww = 0; ww < 2; ++ww) {
                const uint32_t w = words[4 * half + 2 * wp + ww];
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                  // pair (c, c+8): field f = c % 3 of the word shifted by 6 * (c / 3)
                  const int f = c % 3, sh = 6 * (c / 3);
                  const uint32_t v = ((w >> sh) & (fmask << (2 * f))) | 0x43004300u;
                  __nv_bfloat162 p = __hfma2(*reinterpret_cast<const __nv_bfloat162*>(&v), mul[f], add[f]);
                  regs[8 * ww + c] = *reinterpret_cast<uint32_t*>(&p);
                }
              }
              tmem_st16(a_tmem + 16 * wp, regs);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&sm.a_full[ab0]);
            mbar_arrive(&sm.a_full[ab1]);
          }
          hh += 2;
        }
      }
    }
  } else if (warp >= pf::kEpiWarp0) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 168;");
    // ---------------- epilogue: per-group fp32 scale promotion ----------------
    const int e = warp - pf::kEpiWarp0;   // 0..7
    const int q = warp & 3;               // TMEM lane quadrant
    const int cbase = (e >> 2) * TL::kColsPerEpi;  // 0 or BN / 2
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    uint32_t u = 0;
    bool ok = true;
    for (int64_t i = 0, tile; (tile = pf_tile(i, ntiles, n_wt, n_tt, nkc)) >= 0 && ok; ++i) {
      const TileInfo ti = tile_info<BN, KSPLIT>(tile, n_tt, nkc, gpc, ngroups, T, off, S);
      const int64_t n = ti.n0 + 32 * q + lane;
      float2 acc[TL::kColsPerEpi / 2];
#pragma unroll
      for (int c = 0; c < TL::kColsPerEpi / 2; ++c) acc[c] = make_float2(0.0f, 0.0f);
      for (int64_t g = ti.g0; g < ti.g1 && ok; ++g) {
        for (int s = 0; s < ti.kmax; ++s, ++u) {
          // Scale of (slice s, group g, row r) from the staged copy of this unit.
          const uint32_t cs = u % pf::CST, cph = (u / pf::CST) & 1;
          if (!(ok = pf_wait(&sm.c_full[cs], cph, limit, st, 0x332, abort_flag))) break;
          const uint32_t szw = sm.sz[cs][32 * q + lane];
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.c_empty[cs]);
          const float sc = __half2float(__ushort_as_half((unsigned short)(szw & 0xffffu)));
          const float2 sc2 = make_float2(sc, sc);
          const uint32_t db = u % pf::DST, dph = (u / pf::DST) & 1;
          if (!(ok = pf_wait(&sm.d_full[db], dph, limit, st, 0x331, abort_flag))) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem + lane_addr + TL::kTmemD + db * BN + cbase;
          const int lo = (s == 0 ? ti.lo[0] : s == 1 ? ti.lo[1] : s == 2 ? ti.lo[2] : ti.lo[3]) - cbase;  // first active column
          constexpr int CC = TL::kChunkCols;  // columns per wait: CC / 16 loads of 16
#pragma unroll
          for (int cp = 0; cp < TL::kColsPerEpi / CC; ++cp) {
            if (CC * cp + CC <= lo) continue;  // the whole chunk inactive (warp-uniform)
            uint32_t r[CC];
#pragma unroll
            for (int l = 0; l < CC / 16; ++l)
              tmem_ld16(d_tmem + CC * cp + 16 * l, *reinterpret_cast<uint32_t(*)[16]>(&r[16 * l]));
            tmem_ld_wait();
            if (CC * cp >= lo) {  // every column active: packed fp32x2 FMAs
#pragma unroll
              for (int j = 0; j < CC / 2; ++j)
                acc[CC / 2 * cp + j] = __ffma2_rn(sc2, make_float2(__uint_as_float(r[2 * j]),
                                                                   __uint_as_float(r[2 * j + 1])),
                                                  acc[CC / 2 * cp + j]);
            } else {
#pragma unroll
              for (int j = 0; j < CC / 2; ++j) {
                const int c = CC * cp + 2 * j;
                if (c >= lo) acc[CC / 2 * cp + j].x = fmaf(sc, __uint_as_float(r[2 * j]), acc[CC / 2 * cp + j].x);
                if (c + 1 >= lo)
                  acc[CC / 2 * cp + j].y = fmaf(sc, __uint_as_float(r[2 * j + 1]), acc[CC / 2 * cp + j].y);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.d_empty[db]);
        }
      }
      if (!ok) break;
      if (n < N) {
        float* out = Y + (int64_t)ti.kc * T * N;  // chunk kc's partials (the output itself when nkc == 1)
#pragma unroll
        for (int c = 0; c < TL::kColsPerEpi; ++c) {
          const int col = cbase + c;
          if (col < ti.nvalid) {
            const int32_t t = __ldg(perm + ti.t0 + col);
            if (t >= 0 && t < T) out[(int64_t)t * N + n] = (c & 1) ? acc[c >> 1].y : acc[c >> 1].x;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, pf::kTmemCols);
  }
}

// ---- gather: bucket-ordered, swizzled copy of the activations --------------------------
//
// Xt holds, for every (token tile tt, group g), the 48 KB shared-memory image of
// the x tile that the MMA reads: two halves (64 columns each) of 192 rows x 128
// bytes, 16-byte chunk j of row r stored at chunk j ^ (r & 7) (128-byte
// swizzle). Row r of tile tt is the token perm[192 tt + r] (zeros beyond T);
// its permuted column 16w + 2c + e holds x[16w + c + 8e], matching the pair
// order (c, c+8) of a packed word. One thread per 16-column block of a row.
template <int BN>
__global__ void __launch_bounds__(256) prefill_gather_kernel(const __nv_bfloat16* __restrict__ X, int64_t T,
                                                             int64_t K, const int32_t* __restrict__ perm,
                                                             int64_t T_pad, uint8_t* __restrict__ Xt) {
  const int64_t nblk = K / 16;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= T_pad * nblk) return;
  const int64_t i = idx / nblk, w = idx % nblk;
  uint4 a = make_uint4(0, 0, 0, 0), b = a;
  if (i < T) {
    const int32_t src = __ldg(perm + i);
    if (src >= 0 && src < T) {
      const uint4* p = reinterpret_cast<const uint4*>(X + (int64_t)src * K + 16 * w);
      a = __ldg(p);
      b = __ldg(p + 1);
    }
  }
  const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};  // x[0..15] as bf16 pairs
  uint32_t out[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const uint32_t lo = (in[c >> 1] >> (16 * (c & 1))) & 0xffffu;              // x[c]
    const uint32_t hi = (in[(c + 8) >> 1] >> (16 * ((c + 8) & 1))) & 0xffffu;  // x[c + 8]
    out[c] = lo | (hi << 16);
  }
  const int64_t ngroups = K / 128;
  const int64_t tt = i / BN, r = i % BN;
  const int64_t g = w / 8, h = (w % 8) / 4, j0 = 2 * (w % 4);  // chunks j0, j0+1 of half h
  uint8_t* tile = Xt + ((tt * ngroups + g) * 2 + h) * (int64_t)pf::Tile<BN>::kXHalfBytes + r * 128;
  *reinterpret_cast<uint4*>(tile + 16 * ((j0) ^ (r & 7))) = make_uint4(out[0], out[1], out[2], out[3]);
  *reinterpret_cast<uint4*>(tile + 16 * ((j0 + 1) ^ (r & 7))) = make_uint4(out[4], out[5], out[6], out[7]);
}

// ---- host side -------------------------------------------------------------------------

// Tile width and K chunks of a launch: 64-token tiles up to 64 tokens,
// 192-token tiles beyond. K is cut into nkc chunks of equal group counts (none
// empty) when that shortens the launch; the chunk partials are then added by a
// separate reduction. The count minimises a simple cost fitted to
// measurements: the busiest CTA's tiles x (groups per chunk x 3 slices + 4),
// about 1 us per group and slice of a tile plus ~4 us to start and finish a
// tile, plus each chunk's partials written and read back (8 T N bytes at
// 6 TB/s).
struct PfPlan {
  int bn, nkc;
  int64_t T_pad;
  size_t xt_bytes, part_bytes;
};

static PfPlan pf_plan(int64_t T, int64_t N, int64_t K, int sms) {
  PfPlan p;
  const int64_t ngroups = K / 128;
  p.bn = T <= 64 ? 64 : 192;
  p.T_pad = (T + p.bn - 1) / p.bn * p.bn;
  int64_t nkc = 1;
  const int64_t base = ((N + pf::BM - 1) / pf::BM) * ((T + p.bn - 1) / p.bn);
  if (ngroups > 1 && base > 0 && sms > 0) {
    double best = 1e300;
    const int64_t cmax = ngroups < 64 ? ngroups : 64;
    for (int64_t c = 1; c <= cmax; ++c) {
      const int64_t gpc = (ngroups + c - 1) / c, used = (ngroups + gpc - 1) / gpc;
      const int64_t per_cta = (base * used + sms - 1) / sms;
      const double cost = (double)per_cta * ((double)gpc * 3.0 + 4.0) +
                          (used > 1 ? (double)used * 8.0 * (double)T * (double)N / 6.0e6 : 0.0);
      if (cost < best - 1e-9) {
        best = cost;
        nkc = used;
      }
    }
  }
  p.nkc = (int)nkc;
  p.xt_bytes = ((size_t)p.T_pad * (size_t)K * 2 + 255) / 256 * 256;
  p.part_bytes = nkc > 1 ? ((size_t)nkc * (size_t)T * (size_t)N * 4 + 255) / 256 * 256 : 0;
  return p;
}

size_t prefill_ws_bytes(int64_t T, int64_t N, int64_t K) {
  if (T <= 0 || K <= 0) return 256;
  const PfPlan p = pf_plan(T, N, K, num_sms());
  return p.xt_bytes + p.part_bytes;
}

template <int BN, bool KSPLIT>
static cudaError_t launch_prefill_bn(const PfPlan& plan, const void* X, int64_t T, int64_t K, const int32_t* perm,
                                     const int32_t* offsets, const PfCodeMaps& tm_codes, const CUtensorMap& tm_sz,
                                     const uint32_t* sz, int64_t N, int S, float* out, uint8_t* Xt,
                                     cudaStream_t stream, DeviceStatus* st) {
  const int64_t ngroups = K / 128;
  const int64_t blocks_g = (plan.T_pad * (K / 16) + 255) / 256;
  prefill_gather_kernel<BN><<<(unsigned)blocks_g, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(X), T, K,
                                                                   perm, plan.T_pad, Xt);
  auto kernel = prefill_kernel<BN, KSPLIT>;
  const int64_t ntiles = ((N + pf::BM - 1) / pf::BM) * ((T + BN - 1) / BN) * plan.nkc;
  const int grid = (int)(ntiles < num_sms() ? ntiles : num_sms());
  const size_t smem = sizeof(PfSmem<BN>) + 1024;
  cudaError_t e = set_smem((const void*)kernel, (int)smem);
  if (e != cudaSuccess) return e;
  kernel<<<grid, pf::kThreads, smem, stream>>>(Xt, tm_codes, tm_sz, sz, perm, offsets, T, N, ngroups, S, plan.nkc,
                                               out, st, wait_limit());
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, (const void*)kernel);
    char where[160];
    snprintf(where, sizeof where, "prefill launch (%d threads, %d regs/thread, max %d threads, %zu B smem)",
             pf::kThreads, fa.numRegs, fa.maxThreadsPerBlock, smem);
    return note_error(where, e);
  }
  return cudaSuccess;
}

cudaError_t launch_prefill(const void* X, int64_t T, int64_t K, const int32_t* k_t, const int32_t* perm,
                           const int32_t* offsets, const uint32_t* codes, const uint32_t* sz, int64_t N, int S,
                           float* Y, void* ws, cudaStream_t stream, DeviceStatus* st, int bits, int mask1) {
  (void)k_t;
  const int64_t ngroups = K / 128;
  const PfPlan plan = pf_plan(T, N, K, num_sms());
  uint8_t* Xt = static_cast<uint8_t*>(ws);
  float* partial = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + plan.xt_bytes);
  float* out = plan.nkc > 1 ? partial : Y;
  PfCodeMaps tm_codes;
  memset(&tm_codes, 0, sizeof tm_codes);
  CUtensorMap tm_sz;
  if (bits != 3) {  // every slice the same width: one map over all slices
    tm_codes.per_slice = 0;
    tm_codes.mask1 = bits == 1 ? (1 << S) - 1 : 0;
    const uint64_t words = (uint64_t)(K / 32 * bits);  // per row and slice
    if (!make_tmap_2d(&tm_codes.m[0], codes, 4, words, (uint64_t)(S * N), words * 4, (uint32_t)(4 * bits), pf::BM,
                      0))
      return cudaErrorInvalidValue;
  } else {  // one map per slice: slice s starts after the words of slices 0 .. s-1
    tm_codes.per_slice = 1;
    tm_codes.mask1 = mask1;
    const uint32_t* base = codes;
    for (int sl = 0; sl < S; ++sl) {
      const int w = ((mask1 >> sl) & 1) ? 1 : 2;
      const uint64_t words = (uint64_t)(K / 32 * w);
      if (!make_tmap_2d(&tm_codes.m[sl], base, 4, words, (uint64_t)N, words * 4, (uint32_t)(4 * w), pf::BM, 0))
        return cudaErrorInvalidValue;
      base += (size_t)N * words;
    }
  }
  if (!make_tmap_2d(&tm_sz, sz, 4, (uint64_t)N, (uint64_t)(S * ngroups), (uint64_t)N * 4, pf::BM, 1, 0))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (plan.bn == 64)
    e = launch_prefill_bn<64, true>(plan, X, T, K, perm, offsets, tm_codes, tm_sz, sz, N, S, out, Xt, stream, st);
  else if (plan.nkc > 1)
    e = launch_prefill_bn<192, true>(plan, X, T, K, perm, offsets, tm_codes, tm_sz, sz, N, S, out, Xt, stream, st);
  else
    e = launch_prefill_bn<192, false>(plan, X, T, K, perm, offsets, tm_codes, tm_sz, sz, N, S, out, Xt, stream, st);
  if (e != cudaSuccess || plan.nkc <= 1) return e;
  return launch_chunk_reduce(partial, Y, T, N, plan.nkc, stream);
}

}  // namespace mobi
