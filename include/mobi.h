/*
 * mobi.h — C ABI of libmobi: the token-routed mixed-bit linear layer of
 * MoBiQuant on NVIDIA B200 (sm_100a).
 *
 * Sources (the two explainer pages of "MoBiQuant: Mixture-of-Bits Quantization
 * for Token-Adaptive Elastic LLMs"):
 *   [ja]  gist.science/ja/paper/2602.20191 — §2.1 MoBiSlice, §2.2 MoBiRoute
 *   [en]  gist.science/paper/2602.20191 — §2.A MoBiSlice, §2.B MoBiRoute,
 *         §3 Key Contributions (specialised kernels)
 *
 * The layer has three steps and one entry point per step:
 *   mobi_pack   MoBiSlice: W[N,K] -> S residual slices of 2-bit codes with a
 *               per-(slice,row,group) fp16 scale and fp16 zero.
 *               [ja] §2.1 (R_1 = W, W_e = Q(R_e), R_{e+1} = R_e - W_e);
 *               [en] §2.A "Recursive Decomposition" / "Process".
 *   mobi_route  MoBiRoute: k_t = 1 + argmax_j (x_t . Wr[:,j] + b_j), then a
 *               stable bucketing of the tokens by k_t.
 *               [ja] §2.2; [en] §2.B "Routing Mechanism", "Dynamic Adjustment".
 *   mobi_gemm   y_t = x_t . (sum_{s <= k_t} deq(slice_s))^T, fp32 accumulation.
 *               [ja] §2.1 (W^(b) = sum W_e); [en] §2.A "Elasticity".
 * and, built on them:
 *   mobi_linear          routing + GEMM in one call.
 *   mobi_linear_grouped  up to MOBI_MAX_GROUP decode-sized mobi_linear problems
 *                        in one step (mobi_gemm_grouped: the GEMM half).
 *   mobi_route_mlp       threshold routing with a two-layer MLP scorer
 *                        ([ja] §2.2; [en] §2.B "Differentiable Gating").
 *   mobi_pack_bits       generic slicing: 1- or 2-bit slices, wider groups
 *                        (mobi_pack_slices: one width per slice); the GEMM
 *                        entry points' _bits / _slices forms read them.
 *   mobi_ckpt_*          many-in-one checkpoints of packed layers.
 *   mobi_gemm_path, mobi_gemm_decode_noalloc, mobi_sync_check and the size
 *   and status helpers.
 *
 * Conventions shared by every entry point
 *   - Every pointer argument is a DEVICE pointer (allocated by the caller, e.g.
 *     through PyTorch), unless stated otherwise. The library never allocates or
 *     frees device memory; all scratch memory comes from the caller's `ws`.
 *   - Every pointer must be 16-byte aligned (128-bit vector accesses).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls enqueue work and return without synchronising.
 *   - Arguments are validated on the host before anything is launched; on an
 *     error nothing is enqueued and the status says why.
 *   - Supported shapes: S in {1,2,3,4} slices of b = 2 bits (or b = 1 bit
 *     through mobi_pack_bits), group G = 128 along K (256 or 512 through
 *     mobi_pack_bits), K % 128 == 0, N % 16 == 0, T >= 0. K, N, T up to 2^30 elements per
 *     dimension and N*K, T*K, T*N below 2^40.
 *   - A device-side bounded wait that runs out sets a per-device error word;
 *     mobi_sync_check reports it as MOBI_ERR_TIMEOUT (naming the wait site in
 *     mobi_last_error) and clears it.
 *   - Activation range of the decode kernel (every GEMM with T <= 16, and
 *     every grouped or no-alloc call): |x| < 2^31. The kernel feeds x * 2^(96 - 2f)
 *     to the tensor cores as bf16 (so that subnormal code operands stay exact),
 *     which overflows from 2^31 on. A larger |x| (or a NaN/Inf) is not checked
 *     on the host; the kernel flags it and mobi_sync_check returns
 *     MOBI_ERR_INVALID_ARG for that call (its outputs are then unspecified).
 *     The prefill kernel (T > 16) takes any finite bf16.
 *   - The library keeps no per-call host state and is reentrant.
 *
 * Packed format (one checkpoint serves every precision: [ja] §3 "Many-in-One";
 * [en] §3 "MoBiSlice Architecture"). Slices are stored one after another, so a
 * token that needs k slices reads only the first k slices' bytes ([en] §3:
 * bit-major packing avoids the all-or-nothing fetch).
 *
 *   codes  uint32 [S][N][K/16]   word w of (slice s, row n) holds the codes of
 *          k = 16w .. 16w+15; code q(s,n,16w+i) sits in bits [2i+1 : 2i]
 *          (little-endian 2-bit fields). mobi_codes_bytes() gives the size.
 *          1-bit codes (mobi_pack_bits with bits = 1) take 1 bit per weight:
 *          uint32 [S][N][K/32], word w holds k = 32w .. 32w+31 with
 *          q(s,n,32w+i) in bit 2i and q(s,n,32w+16+i) in bit 2i+1 (i < 16): its
 *          even bits are the 2-bit layout's word 2w and its odd bits word
 *          2w+1, each code a 0/1 field. mobi_codes_bytes_bits() gives the size.
 *          Slices of mixed widths (mobi_pack_slices): slice s in the layout of
 *          its width, [N][K*width_s/32] words, the slices one after another
 *          (slice s starts after the words of slices 0..s-1);
 *          mobi_codes_bytes_slices() gives the size.
 *   sz     uint32 [S][K/G][N]    element (s,g,n): bits [15:0] = fp16 scale,
 *          bits [31:16] = fp16 zero (an integer 0..2^b - 1). mobi_sz_bytes().
 *          Group-major so that the scales of one group for consecutive rows
 *          are contiguous (N*4-byte rows, which tensor copies can stage).
 *   The dequantised slice is deq_s[n,k] = (q(s,n,k) - zero(s,n,k/G)) *
 *   scale(s,n,k/G), and the k-slice weight is W^(k) = sum_{s<k} deq_s.
 *
 * Quantiser (the pages name Q(.) but do not define it; this is the reading
 * the library implements, in IEEE fp32 with round-to-nearest-even):
 *   for each (row n, group g):  R <- (float)W[n, group g]
 *   for s = 0..S-1:
 *     mn = min R, mx = max R
 *     sc = max((mx - mn) / 3, 2^-14);  scale = fp16_rne(sc);  s = (float)scale
 *     z  = clamp(rint(-mn / s), 0, 3)
 *     q  = clamp(rint(R / s) + z, 0, 3)          (per element)
 *     R  = R - (q - z) * s                      (the product is exact)
 * Generic slicing (mobi_pack_bits): the same with b-bit codes, L = 2^b - 1
 * steps: sc = max((mx - mn) / L, 2^-14), z and q clamped to [0, L].
 */
#ifndef MOBI_H_
#define MOBI_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOBI_API __attribute__((visibility("default")))
#else
#define MOBI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOBI_OK = 0,
  MOBI_ERR_INVALID_ARG = 1,       /* null pointer, negative size, S/G out of range */
  MOBI_ERR_UNSUPPORTED_SHAPE = 2, /* K % 128, N % 16, or sizes beyond the limits */
  MOBI_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
  MOBI_ERR_WORKSPACE = 4,         /* ws == NULL or ws_bytes below the required size */
  MOBI_ERR_CUDA = 5,              /* a CUDA launch or query failed (error cleared) */
  MOBI_ERR_TIMEOUT = 6,           /* a device-side bounded wait ran out */
  MOBI_ERR_IO = 7                 /* a checkpoint file could not be read or written,
                                     is not one, or failed a checksum */
} mobi_status;

/* Human-readable name of a status (static storage, never NULL). */
MOBI_API const char* mobi_status_string(mobi_status st);

/* Description of the most recent failure seen by a libmobi call on the
 * calling thread (the failing CUDA call or check, and the CUDA error name);
 * empty when none. Static thread-local storage, never NULL. */
MOBI_API const char* mobi_last_error(void);

/* Library version as an integer MAJOR*10000 + MINOR*100 + PATCH. */
MOBI_API int mobi_version(void);

/* Bytes of the packed code array for S slices of an N x K matrix:
 * S * N * (K/16) * 4. Returns 0 for invalid sizes. */
MOBI_API size_t mobi_codes_bytes(int64_t N, int64_t K, int S);
/* Bytes of the codes of S slices of `bits`-bit codes (1 or 2; K % 32 == 0). */
MOBI_API size_t mobi_codes_bytes_bits(int64_t N, int64_t K, int S, int bits);
/* Bytes of the codes of S slices of widths[s]-bit codes (each 1 or 2). */
MOBI_API size_t mobi_codes_bytes_slices(int64_t N, int64_t K, int S, const int* widths);

/* Bytes of the scale/zero array: S * N * (K/G) * 4. Returns 0 for invalid sizes. */
MOBI_API size_t mobi_sz_bytes(int64_t N, int64_t K, int S, int G);

/* Scratch bytes that mobi_route needs for T tokens (may be 0). */
MOBI_API size_t mobi_route_workspace_bytes(int64_t T, int64_t K, int S);

/* Scratch bytes that mobi_gemm needs for exactly this T on the current device
 * (covers both the decode and the prefill kernels, so mobi_gemm_path may pick
 * either). The prefill kernel splits K into chunks when that shortens the
 * launch, and the split depends on T, N, K and the SM count, so the size is
 * not monotone in T: query it for each T used. A smaller buffer is refused
 * with MOBI_ERR_WORKSPACE. */
MOBI_API size_t mobi_gemm_workspace_bytes(int64_t T, int64_t N, int64_t K, int S);

/*
 * mobi_pack — MoBiSlice recursive residual quantisation of W.
 *   [ja] §2.1, [en] §2.A; quantiser as stated at the top of this header.
 *   W        fp16 [N][K] row-major (device). Values must be finite.
 *   N, K     rows and columns; K % G == 0, N % 16 == 0.
 *   G        group size along K; must be 128.
 *   S        number of slices, 1..4.
 *   codes    out, uint32 [S][N][K/16] (layout above).
 *   sz       out, uint32 [S][K/G][N]  (fp16 scale | fp16 zero << 16).
 * Bit-exact with the quantiser above (IEEE division, RNE, no flush-to-zero).
 */
MOBI_API mobi_status mobi_pack(const void* W, int64_t N, int64_t K, int G, int S,
                      uint32_t* codes, uint32_t* sz, void* stream);

/*
 * mobi_pack_bits — MoBiSlice with generic slicing: S slices of `bits`-bit
 *   codes over G-wide groups ([en] §2.A lists 2, 3, 4 or 6-bit precisions;
 *   four 1-bit slices give every width from 1 to 4 bits, three-slice 2-bit
 *   packing only 2, 4 and 6). The quantiser is the one stated at the top of
 *   this header with L = 2^bits - 1 steps.
 *   W, N, K, S, codes  as for mobi_pack (S 1..4; K % G == 0).
 *   G        128, 256 or 512.
 *   bits     1 or 2. 2-bit codes in the 2-bit layout; 1-bit codes at 1 bit per
 *            weight in the 1-bit layout ([en] §3 "Specialized Kernel
 *            Implementation": the bytes fetched follow the bits used), read by
 *            mobi_gemm_bits / mobi_gemm_grouped_bits with bits = 1.
 *   codes    out, mobi_codes_bytes_bits(N, K, S, bits) bytes.
 *   sz       out, uint32 [S][K/128][N] whatever G is: the scale/zero word of
 *            a G-wide group is repeated in each of its G/128 128-column
 *            sub-groups (size: mobi_sz_bytes(N, K, S, 128)), which is the
 *            form the GEMM kernels read.
 * Bit-exact with the quantiser (IEEE division, RNE, no flush-to-zero).
 * Errors: MOBI_ERR_INVALID_ARG for bits outside 1..2, S outside 1..4 or a
 * missing pointer; MOBI_ERR_UNSUPPORTED_SHAPE for other G or K % G != 0.
 */
MOBI_API mobi_status mobi_pack_bits(const void* W, int64_t N, int64_t K, int G, int S, int bits,
                                    uint32_t* codes, uint32_t* sz, void* stream);

/*
 * mobi_pack_slices — mobi_pack_bits with one width per slice: round s of the
 *   recursion quantises the residual with widths[s]-bit codes (1 or 2,
 *   L = 2^widths[s] - 1 steps), and each slice is stored in the layout of its
 *   width, the slices one after another. Widths (2, 1, 1, 2) give 2, 3, 4 and
 *   6 bits per weight from one packed layer, the precisions [en] §2.A lists.
 *   widths   host array of S widths (read during the call only).
 *   codes    out, mobi_codes_bytes_slices(N, K, S, widths) bytes.
 *   Other arguments and errors as for mobi_pack_bits (an invalid width is
 *   MOBI_ERR_INVALID_ARG).
 */
MOBI_API mobi_status mobi_pack_slices(const void* W, int64_t N, int64_t K, int G, int S, const int* widths,
                                      uint32_t* codes, uint32_t* sz, void* stream);

/*
 * mobi_route — MoBiRoute slice count per token and token bucketing.
 *   [ja] §2.2 (a router scores each token; the score fixes how many residual
 *   slices are active); [en] §2.B. The router here is linear:
 *   logit_j(t) = sum_k x[t,k] * Wr[k,j] + bias[j] (fp32 values; the kernel
 *   accumulates in fp32 chunks and fp64 across chunks), and
 *   k_t = 1 + argmax_j logit_j(t), the lowest j winning an exact tie.
 *   X        bf16 [T][K] row-major.
 *   Wr       fp32 [K][S] row-major.  bias  fp32 [S], or NULL for zeros.
 *   k_t      out, int32 [T], values 1..S.
 *   perm     out, int32 [T]: tokens sorted by k_t ascending, stable
 *            (ties keep the original order); perm[i] = original index.
 *   offsets  out, int32 [S+1]: tokens with k_t = j+1 are
 *            perm[offsets[j] .. offsets[j+1]); offsets[0] = 0, offsets[S] = T.
 *   ws       scratch of mobi_route_workspace_bytes(T, K, S) bytes (may be
 *            NULL when that size is 0).
 */
MOBI_API mobi_status mobi_route(const void* X, int64_t T, int64_t K, const float* Wr,
                       const float* bias, int S, int32_t* k_t, int32_t* perm,
                       int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/* Scratch bytes that mobi_route_mlp needs on the current device: the fp32
 * hidden pre-activations of every K split, splits * T * H * 4 rounded up to
 * 256 (the split count depends on T, K, H and the device's SM count; 0 for
 * invalid sizes). */
MOBI_API size_t mobi_route_mlp_workspace_bytes(int64_t T, int64_t K, int64_t H);

/*
 * mobi_route_mlp — threshold routing with a two-layer MLP scorer.
 *   [ja] §2.2: a small MLP scores each token and, at inference, a threshold
 *   turns the gate into a binary mask; moving the threshold trades accuracy
 *   for speed. [en] §2.B "Differentiable Gating" (temperature-scaled sigmoid
 *   gate) and "Dynamic Adjustment" (a larger delta activates fewer slices).
 *   Readings where the pages are silent: a ReLU hidden layer, one score per
 *   residual slice, k_t = 1 + the number of active residual slices:
 *     h_i = max(0, sum_k x[t,k] W1[k,i] + b1[i])       (fp32 accumulation)
 *     s_j = sum_i h_i W2[i,j] + b2[j],   j < S-1       (fp32 accumulation)
 *     slice j+1 active  iff  sigmoid(s_j / tau) > delta,
 *   evaluated as s_j > tau * log(delta / (1 - delta)) in fp64 (the same test,
 *   the sigmoid being increasing).
 *   X        bf16 [T][K] row-major; K % 128 == 0.
 *   W1       fp32 [K][H] row-major.  b1  fp32 [H], or NULL for zeros.
 *   W2       fp32 [H][S-1] row-major. b2  fp32 [S-1], or NULL for zeros.
 *            (W1, W2 may be NULL when S == 1: every k_t is then 1.)
 *   H        hidden width, 1..65536.
 *   tau      temperature, > 0 and finite.  delta  threshold in (0, 1).
 *   k_t, perm, offsets  out, exactly as for mobi_route.
 *   ws       scratch of mobi_route_mlp_workspace_bytes(T, K, H) bytes (may
 *            be NULL for S == 1 or T == 0).
 * Errors: MOBI_ERR_INVALID_ARG for a bad tau, delta, S, H or missing pointer,
 * MOBI_ERR_UNSUPPORTED_SHAPE for K not a multiple of 128 or sizes above the
 * limits, MOBI_ERR_MISALIGNED (X and ws 16-byte, the rest 4-byte aligned),
 * MOBI_ERR_WORKSPACE for a short ws; nothing is launched then.
 */
MOBI_API mobi_status mobi_route_mlp(const void* X, int64_t T, int64_t K, const float* W1,
                                    const float* b1, int64_t H, const float* W2,
                                    const float* b2, int S, double tau, double delta,
                                    int32_t* k_t, int32_t* perm, int32_t* offsets, void* ws,
                                    size_t ws_bytes, void* stream);

/*
 * mobi_gemm — token-routed mixed-bit GEMM.
 *   y[t,n] = sum_k x[t,k] * W^(k_t)[n,k],  W^(k) = sum_{s<k} deq_s,
 *   [ja] §2.1 (W^(b) = sum W_e), [en] §2.A "Elasticity". fp32 accumulation of
 *   exact products: the codes enter the tensor cores as exact small integers
 *   and each slice's fp16 scale is applied in fp32 once per 128-wide group.
 *   X        bf16 [T][K]; k_t, perm, offsets as produced by mobi_route
 *            (k_t values 1..S; perm a permutation sorted by k_t).
 *   codes, sz as produced by mobi_pack for the same N, K, G and >= S slices.
 *   Y        out, fp32 [T][N], original token order.
 *   ws       scratch of mobi_gemm_workspace_bytes(T, N, K, S) bytes.
 * T <= 16 runs the decode kernel (streams only the slices up to the batch's
 * largest k_t), larger T the tcgen05 prefill kernel.
 */
MOBI_API mobi_status mobi_gemm(const void* X, int64_t T, int64_t K, const int32_t* k_t,
                      const int32_t* perm, const int32_t* offsets,
                      const uint32_t* codes, const uint32_t* sz, int64_t N, int G,
                      int S, float* Y, void* ws, size_t ws_bytes, void* stream);

/* Kernel selection for mobi_gemm_path and mobi_gemm_bits. */
typedef enum {
  MOBI_PATH_AUTO = 0,    /* decode for T <= 16, prefill otherwise */
  MOBI_PATH_DECODE = 1,  /* decode kernel; requires T <= 16 */
  MOBI_PATH_PREFILL = 2  /* tcgen05 prefill kernel, any T */
} mobi_path;

/* mobi_gemm with an explicit kernel choice (same arguments and result). */
MOBI_API mobi_status mobi_gemm_path(const void* X, int64_t T, int64_t K, const int32_t* k_t,
                           const int32_t* perm, const int32_t* offsets,
                           const uint32_t* codes, const uint32_t* sz, int64_t N,
                           int G, int S, float* Y, void* ws, size_t ws_bytes,
                           void* stream, int path);

/*
 * mobi_gemm_bits — mobi_gemm_path for slices of `bits`-bit codes (1 or 2, as
 *   written by mobi_pack_bits; 2 is mobi_gemm_path). Same arguments, result
 *   and workspace. Both kernels read each slice's codes in their own layout:
 *   a 1-bit slice streams half the code bytes of a 2-bit one, and the
 *   operands stay exact (a 1-bit code is a 0/1 field where a 2-bit code is a
 *   0..3 field). MOBI_ERR_INVALID_ARG for other widths.
 */
MOBI_API mobi_status mobi_gemm_bits(const void* X, int64_t T, int64_t K, const int32_t* k_t,
                                    const int32_t* perm, const int32_t* offsets, const uint32_t* codes,
                                    const uint32_t* sz, int64_t N, int G, int S, int bits, float* Y, void* ws,
                                    size_t ws_bytes, void* stream, int path);

/*
 * mobi_gemm_slices — mobi_gemm_bits for slices of mixed widths (widths[s]
 *   for slice s, as written by mobi_pack_slices; a host array read during the
 *   call). Every kernel reads each slice in the layout of its width. Same
 *   arguments, result and workspace otherwise; MOBI_ERR_INVALID_ARG for a
 *   width other than 1 or 2.
 */
MOBI_API mobi_status mobi_gemm_slices(const void* X, int64_t T, int64_t K, const int32_t* k_t,
                                      const int32_t* perm, const int32_t* offsets, const uint32_t* codes,
                                      const uint32_t* sz, int64_t N, int G, int S, const int* widths, float* Y,
                                      void* ws, size_t ws_bytes, void* stream, int path);

/* Scratch bytes of mobi_linear: the routing workspace (rounded up to 256
 * bytes) followed by the GEMM workspace. */
MOBI_API size_t mobi_linear_workspace_bytes(int64_t T, int64_t N, int64_t K, int S);

/*
 * mobi_linear — the token-routed mixed-bit linear layer in one call:
 *   mobi_route followed by mobi_gemm on the same stream, with the same
 *   arguments, outputs and results ([ja] §2.2 then §2.1; [en] §2.B then §2.A).
 *   X, Wr, bias, k_t, perm, offsets as for mobi_route; codes, sz, N, G, S, Y
 *   as for mobi_gemm (S is the router's column count as well).
 *   ws       scratch of mobi_linear_workspace_bytes(T, N, K, S) bytes (may be
 *            NULL when that size is 0); the first
 *            align256(mobi_route_workspace_bytes) bytes serve the routing step.
 * What the single call adds: for T <= 16 the decode kernel is launched as a
 * programmatic dependent of the routing kernel, so its launch and set-up
 * overlap the routing (it reads k_t, which decides its work split, only after
 * the routing kernel has finished). Nothing in X, Wr, bias, codes or sz may be
 * written by other work while the call runs. Errors as for mobi_route and mobi_gemm; nothing is
 * launched when an argument is rejected.
 */
MOBI_API mobi_status mobi_linear(const void* X, int64_t T, int64_t K, const float* Wr,
                                 const float* bias, const uint32_t* codes, const uint32_t* sz,
                                 int64_t N, int G, int S, int32_t* k_t, int32_t* perm,
                                 int32_t* offsets, float* Y, void* ws, size_t ws_bytes,
                                 void* stream);

/* mobi_linear for slices of `bits`-bit codes (1 or 2; 2 is mobi_linear), as
 * mobi_gemm_bits is to mobi_gemm_path. */
MOBI_API mobi_status mobi_linear_bits(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                                      const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S, int bits,
                                      int32_t* k_t, int32_t* perm, int32_t* offsets, float* Y, void* ws,
                                      size_t ws_bytes, void* stream);

/* mobi_linear for slices of mixed widths (widths[s] for slice s), as
 * mobi_gemm_slices is to mobi_gemm_path. */
MOBI_API mobi_status mobi_linear_slices(const void* X, int64_t T, int64_t K, const float* Wr, const float* bias,
                                        const uint32_t* codes, const uint32_t* sz, int64_t N, int G, int S,
                                        const int* widths, int32_t* k_t, int32_t* perm, int32_t* offsets,
                                        float* Y, void* ws, size_t ws_bytes, void* stream);

/* One problem of mobi_linear_grouped: the arguments of one mobi_linear call. */
typedef struct mobi_linear_problem {
  const void* X;          /* bf16 [T][K] */
  const float* Wr;        /* fp32 [K][S] */
  const float* bias;      /* fp32 [S], or NULL for zeros */
  const uint32_t* codes;  /* as produced by mobi_pack for N, K */
  const uint32_t* sz;
  float* Y;               /* out, fp32 [T][N] */
  int32_t* k_t;           /* out, int32 [T] */
  int32_t* perm;          /* out, int32 [T] */
  int32_t* offsets;       /* out, int32 [S+1] */
  int64_t T, N, K;
} mobi_linear_problem;

/* Largest problem count of one mobi_linear_grouped call. */
#define MOBI_MAX_GROUP 16

/* Scratch bytes of mobi_linear_grouped for these problems (0 for invalid
 * arguments or when none is needed). */
MOBI_API size_t mobi_linear_grouped_workspace_bytes(const mobi_linear_problem* problems, int count,
                                                    int S);

/* One problem of mobi_gemm_grouped: the arguments of one decode-sized mobi_gemm. */
typedef struct mobi_gemm_problem {
  const void* X;          /* bf16 [T][K] */
  const int32_t* k_t;     /* int32 [T], values 1..S */
  const uint32_t* codes;  /* as produced by mobi_pack for N, K */
  const uint32_t* sz;
  float* Y;               /* out, fp32 [T][N] */
  int64_t T, N, K;
} mobi_gemm_problem;

/* Scratch bytes of mobi_gemm_grouped (0 for invalid arguments or none needed). */
MOBI_API size_t mobi_gemm_grouped_workspace_bytes(const mobi_gemm_problem* problems, int count, int S);

/*
 * mobi_gemm_grouped — the GEMM half of mobi_linear_grouped: up to
 *   MOBI_MAX_GROUP decode-sized (T <= 16) mobi_gemm problems whose k_t are
 *   already known, one decode launch per fragment class plus one chunk
 *   reduction. Results equal one mobi_gemm call per problem bit for bit.
 *   Errors as for mobi_gemm, checked for every problem before any launch.
 */
MOBI_API mobi_status mobi_gemm_grouped(const mobi_gemm_problem* problems, int count, int G, int S,
                                       void* ws, size_t ws_bytes, void* stream);

/* mobi_gemm_grouped for slices of `bits`-bit codes (1 or 2; every problem of
 * the call has that width), as mobi_gemm_bits is to mobi_gemm_path. */
MOBI_API mobi_status mobi_gemm_grouped_bits(const mobi_gemm_problem* problems, int count, int G, int S, int bits,
                                            void* ws, size_t ws_bytes, void* stream);

/* mobi_gemm_grouped for slices of mixed widths (every problem of the call has
 * the widths `widths`). */
MOBI_API mobi_status mobi_gemm_grouped_slices(const mobi_gemm_problem* problems, int count, int G, int S,
                                              const int* widths, void* ws, size_t ws_bytes, void* stream);

/*
 * mobi_linear_grouped — up to MOBI_MAX_GROUP independent decode-sized
 *   mobi_linear problems (every T <= 16) in one step: the projections of a
 *   layer that read their weights in the same decode step ([en] §3: only the
 *   slices needed are fetched, so the step is bound by weight bytes; the
 *   explainer pages' deployment discussion of one model serving many
 *   precisions). Each problem's results are exactly those of mobi_linear on
 *   it alone (same kernels, same summation order).
 *   problems  host array of `count` descriptors (1..MOBI_MAX_GROUP); the
 *             library reads it during the call only.
 *   G, S      group size (128) and slice count, shared by all problems.
 *   ws        scratch of mobi_linear_grouped_workspace_bytes bytes.
 * Launches: one routing launch (an 8-CTA cluster per problem), one decode
 * launch per fragment class present (T <= 8 and 9..16 tokens; the SMs are
 * shared among that class's problems in equal parts of the slice bytes they
 * read, once k_t is known), and one chunk-reduction launch, so per-launch
 * ramp-up and drain are paid once per step instead of once per problem. Outputs must not overlap any
 * problem's inputs or each other. Errors as for mobi_linear, checked for every
 * problem before anything is launched; T > 16 gives MOBI_ERR_UNSUPPORTED_SHAPE.
 */
MOBI_API mobi_status mobi_linear_grouped(const mobi_linear_problem* problems, int count, int G,
                                         int S, void* ws, size_t ws_bytes, void* stream);

/* mobi_linear_grouped for slices of `bits`-bit codes (1 or 2; every problem of
 * the call has that width). */
MOBI_API mobi_status mobi_linear_grouped_bits(const mobi_linear_problem* problems, int count, int G, int S,
                                              int bits, void* ws, size_t ws_bytes, void* stream);

/* mobi_linear_grouped for slices of mixed widths (every problem of the call
 * has the widths `widths`). */
MOBI_API mobi_status mobi_linear_grouped_slices(const mobi_linear_problem* problems, int count, int G, int S,
                                                const int* widths, void* ws, size_t ws_bytes, void* stream);

/* ---- many-in-one checkpoints of packed layers -------------------------------
 *
 * One file holds the packed slices of any number of layers ([ja] §2.1: a single
 * decomposition serves every precision; [en] §3: "many-in-one" storage, only
 * the slices needed are fetched). Because codes and scale/zero words are
 * slice-major, loading a layer at k slices (2k bits) reads only the first k
 * slices of each block: a prefix of the file's codes block and of its sz block.
 *
 * File format (little-endian; version 1):
 *   [0, 64)  header: "MOBICKPT", u32 version, u32 count, u64 table offset,
 *            u64 table bytes, u32 CRC-32C of the table, 28 reserved bytes.
 *   table    count entries of 192 bytes: name (96 bytes, NUL-terminated),
 *            i64 N, i64 K, i32 G, i32 S, u64 codes offset, u64 codes bytes per
 *            slice (N K / 4), u64 sz offset, u64 sz bytes per slice (K/G N 4),
 *            u32 CRC-32C of each slice's codes [4] and sz [4], zero padding.
 *   data     per tensor its codes block [S][N][K/16] u32 and its sz block
 *            [S][K/G][N] u32, each starting on a 4096-byte boundary.
 * CRC-32C is the Castagnoli CRC (reflected polynomial 0x82F63B78, initial
 * value and final xor 0xFFFFFFFF).
 *
 * host_ptrs = 1: codes and sz are host memory; 0: device memory (copied
 * through pinned staging buffers on `stream`; the call returns once the data
 * has arrived). Errors: MOBI_ERR_INVALID_ARG (bad argument, duplicate or
 * over-long name, index or slice count out of range), MOBI_ERR_IO (file
 * errors, bad magic or version, truncated file, checksum mismatch),
 * MOBI_ERR_CUDA (a copy failed). A failed save leaves no file at `path`.
 */
typedef struct mobi_ckpt_tensor {
  const char* name;       /* at most 95 bytes, unique in the file */
  const uint32_t* codes;  /* [S][N][K/16], as produced by mobi_pack (2-bit codes only) */
  const uint32_t* sz;     /* [S][K/G][N] */
  int64_t N, K;
  int G, S;
} mobi_ckpt_tensor;

typedef struct mobi_ckpt mobi_ckpt; /* an open checkpoint (not thread-safe) */

/* Write `count` packed tensors to `path` (written to a temporary name, then
 * renamed). */
MOBI_API mobi_status mobi_ckpt_save(const char* path, const mobi_ckpt_tensor* tensors, int count,
                                    int host_ptrs, void* stream);
/* Open a checkpoint: reads and checks the header and the table. */
MOBI_API mobi_status mobi_ckpt_open(const char* path, mobi_ckpt** out);
/* Number of tensors; -1 for NULL. */
MOBI_API int mobi_ckpt_count(const mobi_ckpt* ckpt);
/* Index of the tensor called `name`, or -1. */
MOBI_API int mobi_ckpt_find(const mobi_ckpt* ckpt, const char* name);
/* Shape of tensor `index`; *name points into the reader (valid until close). */
MOBI_API mobi_status mobi_ckpt_info(const mobi_ckpt* ckpt, int index, const char** name, int64_t* N,
                                    int64_t* K, int* G, int* S);
/* Load the first `slices` slices (1..S) of tensor `index` into codes
 * [slices][N][K/16] and sz [slices][K/G][N]: a packed array with S = slices.
 * verify = 1 checks the CRC of every slice read. */
MOBI_API mobi_status mobi_ckpt_load(mobi_ckpt* ckpt, int index, int slices, uint32_t* codes,
                                    uint32_t* sz, int host_ptrs, int verify, void* stream);
/* Bytes read from the file by this reader so far (data blocks only). */
MOBI_API int64_t mobi_ckpt_bytes_read(const mobi_ckpt* ckpt);
/* Close the reader (NULL is a no-op). */
MOBI_API void mobi_ckpt_close(mobi_ckpt* ckpt);
/* CRC-32C of n bytes of host memory, continuing from `crc` (0 to start). */
MOBI_API uint32_t mobi_crc32c(uint32_t crc, const void* data, size_t n);

/*
 * mobi_gemm_decode_noalloc — the decode GEMM (T <= 16) without a workspace.
 *   Not part of the method: the MoBiQuant pages have no counterpart of this
 *   call. It exists for callers that cannot allocate device memory at launch
 *   time: an engine plugin whose enqueue step must not allocate, a real-time
 *   loop that runs under a fixed memory budget, or a host whose device memory
 *   belongs to another runtime that only hands out input and output buffers.
 *   Such callers cannot provide the workspace that mobi_gemm needs.
 *   Same arguments and result as mobi_gemm for T <= 16, minus perm, offsets
 *   and the workspace: the scratch lives in one 8 MiB array of static device
 *   memory that every GPU loading this library holds until the process exits.
 *   Shapes whose decode scratch exceeds 8 MiB (mobi_gemm_workspace_bytes
 *   larger than 8 MiB, e.g. N * ceil(K/1024) * 64 bytes beyond it) are
 *   rejected with MOBI_ERR_WORKSPACE before anything is launched.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents, so calls that overlap on the GPU (other streams, other host
 *   threads) race: serialise them. The call itself allocates nothing.
 */
MOBI_API mobi_status mobi_gemm_decode_noalloc(const void* X, int64_t T, int64_t K, const int32_t* k_t,
                                              const uint32_t* codes, const uint32_t* sz, int64_t N, int G,
                                              int S, float* Y, void* stream);

/*
 * mobi_sync_check — synchronise `stream`, then report and clear the
 * device-side error word of the current device. Returns MOBI_ERR_TIMEOUT if a
 * bounded wait ran out since the last check (mobi_last_error names the wait
 * site), MOBI_ERR_INVALID_ARG if a decode call met an activation with
 * |x| >= 2^31 (see the activation range above), MOBI_ERR_CUDA on a CUDA error,
 * MOBI_OK otherwise.
 */
MOBI_API mobi_status mobi_sync_check(void* stream);

/*
 * mobi_debug_set_wait_limit — set the iteration limit of the device-side
 * bounded waits of the current device (0 restores the default). A tiny limit
 * makes the kernels' waits run out, which exercises the timeout path without
 * faulting anything: the kernel records the error, drains its own copies (and
 * MMAs) in flight, frees its tensor memory and returns. Below 64 the decode
 * kernel's waits poll without suspending and each of its warps first waits on
 * a barrier that nothing completes, so its timeout path always runs.
 * Test use only.
 */
MOBI_API mobi_status mobi_debug_set_wait_limit(int64_t limit);

#ifdef __cplusplus
}
#endif

#endif /* MOBI_H_ */
