/*
 * rbq.h -- C ABI of the B200 rotate-then-quantize library (librbq.so).
 *
 * The library implements the data-parallel hot path of rotation-based
 * post-training quantisation for diffusion-transformer linear layers:
 *
 *   OrbitQuant (write-up at hotelren.com/news/3376620):
 *     §2.3  the random-permuted block-Hadamard rotation (RPBH)
 *           Pi_d = blkdiag(H_64 D_1, ..., H_64 D_{d/64}) · P_pi;
 *     §1, §4.2  one Lloyd-Max codebook per input width d for N(0, 1/d);
 *     §2.1  offline weights: W' = W Pi^T, row norms r' (BF16), direction codes;
 *     §2.2  online activations: x' = Pi x, norm s, direction codes; the rotation
 *           cancels inside the linear, y = r' s sum_k C_w[q] C_a[p].
 *   INT8-convrot ("INT8旋转量化是什么", cloud.baidu.com/article/9430339) §4 and
 *   the rotated-model explainer (cloud.baidu.com/article/9432521) §4:
 *     rotate, then symmetric INT8 with a per-output-channel scale; inference
 *     either dequantises or runs an INT8 operator (here: W8A16).
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor arguments are DEVICE pointers to memory the caller allocated
 *   (for example with PyTorch); the library never frees them.  Row-major,
 *   no padding between rows.
 * - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *   stream).  Kernel calls are asynchronous on that stream; there is no hidden
 *   device-wide synchronisation.
 * - The return value is RBQ_OK (0) or a negative RBQ_E* code.  Arguments are
 *   validated before anything is launched, so a call that returns
 *   RBQ_EINVAL / RBQ_EALIGN has written nothing.  RBQ_ECUDA reports a failed
 *   launch or allocation inside the library; rbq_error_string() names it.
 * - The first compute call that uses an RPBH handle or a (d, bits) codebook on
 *   a device uploads small tables to that device synchronously (a few KB).
 *   Make that first call before capturing a stream into a CUDA graph.
 * - Dense inputs are BF16 (RBQ_BF16) or fp32 (RBQ_F32), d a multiple of 64.
 * - Packed codes: code j of a row occupies bits [j*b, j*b+b) of the row's
 *   little-endian bitstream (LSB first); the row pitch is d*b/8 bytes.
 *   (The pages do not fix a bit layout; this is the library's.)
 */
#ifndef RBQ_H
#define RBQ_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- return codes ------------------------------------------------------ */
#define RBQ_OK          0
#define RBQ_EINVAL     (-1)  /* bad size, bit width, mode, dtype or NULL pointer */
#define RBQ_EALIGN     (-2)  /* pointer not aligned as documented               */
#define RBQ_ECUDA      (-3)  /* CUDA launch / allocation / copy failed          */
#define RBQ_ENOMEM     (-4)  /* host allocation failed                          */
#define RBQ_ECONVERGE  (-5)  /* Lloyd-Max solver did not converge               */
#define RBQ_EDEVICE    (-6)  /* kernel reported an internal error (see below)   */
#define RBQ_ESCRATCH   (-7)  /* problem larger than a fixed scratch area        */
#define RBQ_EIO        (-8)  /* layer file: open/read/write failed or not valid */

/* ---- element types and modes --------------------------------------------- */
#define RBQ_F32    0
#define RBQ_BF16   1

#define RBQ_LLOYDMAX   0   /* OrbitQuant direction codes + BF16 row norms     */
#define RBQ_INT8_SYM   1   /* symmetric per-output-channel INT8 + fp32 scales */
#define RBQ_INT8_TENSOR 2  /* symmetric INT8, one scale for the whole tensor   */

#define RBQ_ROTATE_ONLY 16 /* `bits` value of rotate_quantize_act: x' only  */

/* ---- RPBH transform (OrbitQuant §2.3) ------------------------------------ */

/* Opaque handle: the permutation pi and signs D of one Pi_d, on the host and
 * (after first use) on each device that used it. */
typedef struct rbq_rpbh rbq_rpbh;

/*
 * rpbh_make -- draw Pi_d = blkdiag(H_h D_1 ... H_h D_{d/h}) · P_pi from `seed`.
 *   d     input width, a positive multiple of h, at most 32768
 *   h     Hadamard block size; must be 64
 *   seed  any 64-bit value
 *   out   receives the new handle (free with rpbh_free)
 * The draw is fixed by this library (the pages ask only that it be
 * reproducible across platforms, OrbitQuant §6.3): SplitMix64 started at
 * `seed`; Fisher-Yates for i = d-1..1 with j = floor(u*(i+1)/2^64); then d
 * sign draws, D_k = -1 when the top bit is set.  (P_pi x)_k = x_{pi(k)}.
 * H_h is the Sylvester-order Walsh-Hadamard matrix scaled by 1/sqrt(h).
 * Host only: works without a GPU.  Errors: RBQ_EINVAL, RBQ_ENOMEM.
 */
int rpbh_make(int d, int h, uint64_t seed, rbq_rpbh** out);

/*
 * rpbh_make_ablation -- the same draw with parts of Pi_d switched off, for the
 * ablations the OrbitQuant write-up reports (§3.3; §2.3 gives the reason for
 * P_pi: without it outliers can stay concentrated in some blocks, with it
 * every coordinate's variance is close to 1/d).  The random stream is consumed exactly
 * as by rpbh_make, so with flags = 0 the result equals rpbh_make's and the
 * signs of an RBQ_RPBH_NO_PERMUTATION handle equal the full draw's.
 *   flags  RBQ_RPBH_NO_PERMUTATION: pi = identity (block Hadamard with D)
 *          RBQ_RPBH_NO_SIGNS:       D = +1
 * The handle is used like any other (every kernel takes it).
 * Host only.  Errors: RBQ_EINVAL (also for unknown flag bits), RBQ_ENOMEM.
 */
#define RBQ_RPBH_NO_PERMUTATION 1
#define RBQ_RPBH_NO_SIGNS       2
int rpbh_make_ablation(int d, int h, uint64_t seed, int flags, rbq_rpbh** out);

/* rpbh_free -- release a handle and its device copies (NULL is a no-op).
 * The caller must ensure no launched kernel still uses it. */
void rpbh_free(rbq_rpbh* r);

/* rpbh_export -- copy pi (int32[d]) and D (int8[d], +-1) to HOST buffers.
 * Either pointer may be NULL.  Errors: RBQ_EINVAL. */
int rpbh_export(const rbq_rpbh* r, int32_t* perm_host, int8_t* signs_host);

/* rpbh_describe -- the transform info that rebuilds the handle exactly:
 * rpbh_make_ablation(d, h, seed, flags) draws the same pi and D.  Any output
 * pointer may be NULL.  Errors: RBQ_EINVAL. */
int rpbh_describe(const rbq_rpbh* r, int* d, int* h, uint64_t* seed, int* flags);

/* rpbh_dim -- d of a handle, or RBQ_EINVAL for NULL. */
int rpbh_dim(const rbq_rpbh* r);

/* ---- Lloyd-Max codebook (OrbitQuant §1, §4.2) ---------------------------- */

/*
 * lloydmax_table -- MSE-optimal 2^bits-level quantiser of N(0, 1/d).
 *   d       input width (> 0); the table is the N(0,1) table times 1/sqrt(d)
 *   bits    1..8
 *   levels  HOST double[2^bits], increasing, antisymmetric (may be NULL)
 *   bounds  HOST double[2^bits - 1], the midpoints of adjacent levels; the
 *           middle one is exactly 0 (may be NULL)
 * Solved in fp64 by Newton's method on the centroid/midpoint conditions.
 * Host only.  Errors: RBQ_EINVAL, RBQ_ECONVERGE.
 */
int lloydmax_table(int d, int bits, double* levels, double* bounds);

/* ---- rotate-then-quantise kernels ---------------------------------------- */

/*
 * rotate_quantize_act -- online activation quantiser (OrbitQuant §2.2),
 * one fused kernel per call.  For every token row x of X[T, d]:
 *   x' = Pi_d x;  s = ||x'||_2 (fp32);  v = x' / (s + 1e-12);
 *   code_k = #{ j : t_j <= v_k }  over the Lloyd-Max boundaries of (d, bits)
 *            (nearest level, ties to the upper level);
 *   codes row = packed codes (LSB-first bitstream, d*bits/8 bytes).
 *   r       RPBH handle of width d
 *   X       device, T x d, dtype RBQ_BF16 or RBQ_F32, 16-byte aligned
 *   T       number of tokens (0 is a valid no-op)
 *   bits    1..8, or RBQ_ROTATE_ONLY: then `codes_out` receives x' itself as
 *           BF16 [T, d] (round to nearest even) -- the activation operand of
 *           qlinear_int8 -- and `norms_out` may be NULL
 *   codes_out  device, T x (d*bits/8) bytes, 16-byte aligned
 *   norms_out  device float[T], s per token, 4-byte aligned
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int rotate_quantize_act(const rbq_rpbh* r, const void* X, int dtype, int T,
                        int bits, void* codes_out, float* norms_out,
                        void* stream);

/*
 * quantize_weights -- offline weight quantiser, the same fused kernel run on
 * the d_out rows of W[d_out, d] (each row w_i becomes w'_i = Pi_d w_i, i.e.
 * W' = W Pi^T, OrbitQuant §2.1).
 *   mode RBQ_LLOYDMAX: bits 1..8; `codes_or_q` = packed direction codes
 *        (d_out x d*bits/8 bytes); `rownorm_or_scale` = uint16 BF16 r'_i =
 *        bf16(||w'_i||) (round to nearest even).  Directions are w'/(r + 1e-12)
 *        with the fp32 norm r.
 *   mode RBQ_INT8_SYM: bits must be 8; `codes_or_q` = int8 q [d_out, d];
 *        `rownorm_or_scale` = float scale_i = max_k |w'_ik| / 127;
 *        q = clamp(round_half_even(w' / scale), -127, 127); a zero row gives
 *        scale 0 and q 0 (INT8-convrot §4; the zero point is 0).
 *   mode RBQ_INT8_TENSOR: as RBQ_INT8_SYM with one scale for the whole
 *        tensor, S = max_ik |w'_ik| / 127 (the INT8 image-text model page,
 *        cloud.baidu.com/article/9432337, "how it works": one scale per
 *        tensor), written to every entry of `rownorm_or_scale` so that
 *        qlinear_int8 takes it unchanged.  Two passes over W: per-row maxima
 *        (then their maximum), then the rows quantised with S.
 *   W  device, d_out x d, dtype RBQ_BF16 or RBQ_F32, 16-byte aligned.
 *   Output pointers 16-byte (codes/q) and 4-byte (norms/scales) aligned.
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int quantize_weights(const rbq_rpbh* r, const void* W, int dtype, int d_out,
                     int mode, int bits, void* codes_or_q,
                     void* rownorm_or_scale, void* stream);

/*
 * quantize_weights_int8_asym -- asymmetric per-output-channel INT8 with a zero
 * point (INT8-convrot, "the quantized model file": scale and zero point per
 * layer/channel; the INT8 image-text model page, "how it works").  For each
 * row w'_i = Pi_d w_i:
 *   hi = max(max_k w'_ik, 0), lo = min(min_k w'_ik, 0), scale_i = (hi - lo)/255,
 *   z_i = clamp(round_half_even(-lo / scale_i), 0, 255),
 *   q_ik = clamp(round_half_even(w'_ik / scale_i) + z_i, 0, 255);
 *   w'_ik ~ scale_i (q_ik - z_i); a zero row gives scale 0, z 0, q 0.
 *   W           device, d_out x d, RBQ_BF16 or RBQ_F32, 16-byte aligned
 *   q           device uint8 [d_out, d], 16-byte aligned
 *   scale       device float [d_out], 4-byte aligned
 *   zero_point  device uint8 [d_out]
 * Offline weights: runs the general rotation kernel (any width).
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int quantize_weights_int8_asym(const rbq_rpbh* r, const void* W, int dtype, int d_out, uint8_t* q, float* scale,
                               uint8_t* zero_point, void* stream);

/* ---- quantised linear layers --------------------------------------------- */

/*
 * qlinear -- OrbitQuant §2.2 (the rotation cancels):
 *   Y[m, n] = bf16( s[m] * r'[n] * sum_k C_w[q[n,k]] * C_a[p[m,k]] ),
 * with C_a / C_w the Lloyd-Max levels of (K, bits_a) / (K, bits_w), operands
 * expanded on the fly into tensor-core tiles, fp32 accumulation.
 *   a_codes  device, M x (K*bits_a/8) bytes, from rotate_quantize_act
 *   s        device float[M], norms from rotate_quantize_act
 *   w_codes  device, N x (K*bits_w/8) bytes, from quantize_weights
 *   rnorm    device uint16 BF16[N], row norms from quantize_weights
 *   M, N, K  tokens, output width, input width (K a multiple of 64)
 *   Y        device uint16 BF16 [M, N], row-major
 * Alignment: code arrays 16-byte, Y 16-byte, s/rnorm 4-byte.
 * Workspace (K a multiple of 128, N of 8, 16-byte code rows): the weight codes
 * are expanded per call into fp16 levels, N*K*2 bytes from a stream-ordered
 * memory pool, and the activation codes too, M*K*2 more bytes, while that
 * part is at most 2 GiB (beyond it the GEMM expands them itself).  Other
 * shapes run a general kernel that expands both operands tile by tile
 * without a workspace.
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int qlinear(const uint8_t* a_codes, const float* s, int bits_a,
            const uint8_t* w_codes, const uint16_t* rnorm, int bits_w,
            int M, int N, int K, uint16_t* Y, void* stream);

/*
 * qlinear_int8 -- W8A16 linear of the INT8 path (INT8-convrot §4):
 *   Y[m, n] = bf16( scale[n] * sum_k q[n,k] * Xrot[m,k] ),
 * Xrot = bf16(Pi x) from rotate_quantize_act(bits = RBQ_ROTATE_ONLY), q and
 * scale from quantize_weights(RBQ_INT8_SYM).  fp32 accumulation.
 *   Xrot   device uint16 BF16 [M, K];  Wq device int8 [N, K];
 *   scale  device float[N];  Y device uint16 BF16 [M, N]
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int qlinear_int8(const uint16_t* Xrot, const int8_t* Wq, const float* scale,
                 int M, int N, int K, uint16_t* Y, void* stream);

/*
 * qlinear_int8_levels -- the quantised linear layer with each codebook's
 * levels rounded onto a signed 8-bit grid, run on the INT8 tensor cores
 * (tcgen05 kind::i8) with exact int32 accumulation.  A deployment variant of
 * qlinear (OrbitQuant §2.2, "Online inference": the same codes, norms and
 * cancellation) for 8-bit integer tensor cores, the kind of low-precision
 * operator OrbitQuant §4.2-§4.4 points deployments to (start from W8A8, then
 * lower the widths); the pages do not define it, so its result is its own:
 *   l_b[j] = RNE(alpha_b * c_j),  alpha_b = 127 / max_j |c_j|   (int8 levels)
 *   Y[m, n] = bf16( s[m] * r'[n] * (sum_k l_w[q_nk] * l_a[p_mk]) / (alpha_w * alpha_a) )
 * with c_j the N(0, 1/K) Lloyd-Max levels of lloydmax_table(K, bits); the
 * integer sum is exact, the scaling is fp32.  rbq_int8_levels returns l and
 * alpha.  Arguments, layouts and ownership as qlinear.
 * Limits: K a multiple of 128, N a multiple of 8, K*bits_a/8 a multiple of
 * 16 (else RBQ_EINVAL; there is no fallback kernel).
 * The weight and activation codes are expanded once per call into an int8
 * workspace of (N + M)*K bytes from a stream-ordered memory pool.
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECONVERGE, RBQ_ECUDA.
 */
int qlinear_int8_levels(const uint8_t* a_codes, const float* s, int bits_a,
                        const uint8_t* w_codes, const uint16_t* rnorm, int bits_w,
                        int M, int N, int K, uint16_t* Y, void* stream);

/*
 * qlinear_fp8_levels -- the same layer with each codebook's levels rounded to
 * FP8 E4M3 (OCP E4M3FN, round to nearest even) and summed in fp32 on the FP8
 * tensor cores (tcgen05 kind::f8f6f4):
 *   e_b[j] = E4M3(beta_b * c_j),  beta_b = 2^(7 - floor(log2 max_j |c_j|))
 *   Y[m, n] = bf16( s[m] * r'[n] * (sum_k e_w[q_nk] * e_a[p_mk]) / (beta_w * beta_a) )
 * beta is a power of two, so the levels lose only their mantissa bits beyond
 * the third (relative error <= 2^-4); the sum is fp32 (not exact).
 * rbq_fp8_levels returns the E4M3 bytes and beta.  Arguments, layouts, limits,
 * workspace and errors as qlinear_int8_levels.
 */
int qlinear_fp8_levels(const uint8_t* a_codes, const float* s, int bits_a,
                       const uint8_t* w_codes, const uint16_t* rnorm, int bits_w,
                       int M, int N, int K, uint16_t* Y, void* stream);

/*
 * rbq_fp8_levels -- the E4M3 levels qlinear_fp8_levels uses for (d, bits)
 * (host only): levels HOST uint8[2^bits] E4M3 bytes (may be NULL), beta HOST
 * double (may be NULL).  Returns RBQ_OK, RBQ_EINVAL or RBQ_ECONVERGE.
 */
int rbq_fp8_levels(int d, int bits, uint8_t* levels, double* beta);

/*
 * rbq_int8_levels -- the integer levels qlinear_int8_levels uses for (d, bits)
 * (host only): levels HOST int8[2^bits] (may be NULL), alpha HOST double
 * (may be NULL).  Returns RBQ_OK, RBQ_EINVAL or RBQ_ECONVERGE.
 */
int rbq_int8_levels(int d, int bits, int8_t* levels, double* alpha);

/*
 * qlinear_noalloc -- the same result as qlinear, for callers that cannot
 * allocate device memory.  (The pages have no counterpart: this is a
 * deployment variant of the library, not a step of the method.)
 *
 * qlinear expands the weight codes (and, at activation widths other than 4
 * bits, the activation codes) into an fp16 workspace taken from a
 * stream-ordered memory pool on every call.  Callers that own all device
 * memory through their own allocator, forbid allocation on their inference
 * thread, or run inside a process whose allocator is not CUDA's cannot accept
 * that.  This entry point allocates nothing: its workspace, 16 slots for
 * level tables and a fallback error word live in one fixed __device__ array
 * of 32 MiB + 8448 bytes inside the library, which every GPU that loads the
 * library holds until the process exits.
 *   Arguments as qlinear, plus
 *   err   device uint32 the kernels OR a non-zero value into when a bounded
 *         pipeline wait runs out (Y is then invalid); caller-owned, the caller
 *         clears it; NULL = record in the array's own word (not reported).
 * Limits: N*K <= 16,777,216 (else RBQ_ESCRATCH, nothing launched); K a
 * multiple of 128, N a multiple of 8, K*bits_a/8 a multiple of 16 (else
 * RBQ_EINVAL).
 * Set-up happens inside calls: the first call on a device looks up the
 * array's device address (cudaGetSymbolAddress, with that device current),
 * and the first call on a device for each (K, bits) pair copies that level
 * table from host memory into a free slot of the array, ordered on the call's
 * stream before its kernels (with all 16 slots taken, slots are reused in
 * turn).  Make those first calls before any stream capture; later calls with
 * widths already in a slot launch the two kernels and copy nothing.  Every
 * call uses the same array and the array keeps the last call's contents, so
 * calls whose work overlaps on the GPU (on different streams, or from several
 * host threads) race and corrupt each other's results; serialise them on one
 * stream.  Nothing in the array needs to start at zero: a slot is written
 * before its first use and each call's expansion writes every workspace
 * element its GEMM reads.
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ESCRATCH, RBQ_ECONVERGE, RBQ_ECUDA.
 */
int qlinear_noalloc(const uint8_t* a_codes, const float* s, int bits_a,
                    const uint8_t* w_codes, const uint16_t* rnorm, int bits_w,
                    int M, int N, int K, uint16_t* Y, unsigned int* err,
                    void* stream);

/* ---- diagnostics ----------------------------------------------------------- */

/*
 * rbq_code_grid -- a code-search table the kernels use for (d, bits), for
 * inspection and tests (host only).  A coordinate v gets
 *   n = round_to_nearest( clamp(v * scale + 0.5, 0, 1) * cells ),
 *   code = base[n] + (v >= thr[n]),
 * which equals #{ j : t_j <= v } outside a rounding band around each boundary.
 *   variant  0: grid over [-R, R] just wider than the outermost boundary
 *               (the kernels clamp); 1: grid over [-1, 1], the range of a unit
 *               vector's coordinates (no clamp; RBQ_ECONVERGE when it would
 *               exceed 5000 cells)
 *   thr    HOST float[cells + 1] (may be NULL)
 *   base   HOST int32[cells + 1] (may be NULL)
 *   cells, scale  receive the grid size and the factor 1/(2R)
 * Returns RBQ_OK, RBQ_EINVAL or RBQ_ECONVERGE.
 */
int rbq_code_grid(int d, int bits, int variant, float* thr, int32_t* base, int* cells, float* scale);

/*
 * qlinear_int8_asym -- the W8A16 layer on asymmetric INT8 weights:
 *   Y[m, n] = bf16( scale[n] * sum_k (q[n,k] - z[n]) * Xrot[m,k] ),
 * fp32 accumulation.  The weights are widened once per call to bf16 (q - z),
 * which is exact, and run through the same tensor-core GEMM as qlinear_int8.
 *   Xrot        device BF16 [M, K] from rotate_quantize_act(bits=RBQ_ROTATE_ONLY)
 *   q, scale, zero_point  from quantize_weights_int8_asym
 *   N a multiple of 8, K a multiple of 64 (else RBQ_EINVAL); Y BF16 [M, N].
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int qlinear_int8_asym(const uint16_t* Xrot, const uint8_t* Wq, const float* scale, const uint8_t* zero_point,
                      int M, int N, int K, uint16_t* Y, void* stream);

/* ---- the rotation fused into the producing matmul ---------------------------
 * OrbitQuant §6.2 ("performance below expectations") points at fusing the
 * rotation with the matrix-multiply kernels to cut memory traffic.  The
 * rotation of a layer's input gathers it by pi across the whole row, which no
 * output tile of the producing GEMM holds; with the producing layer's weight
 * rows reordered offline by that pi, each 64 consecutive output columns are
 * the inputs of one Hadamard block, and the producing GEMM's epilogue can
 * finish the rotation. */
#define RBQ_ACT_NONE 0
#define RBQ_ACT_GELU 1   /* exact GELU: y Phi(y) = 0.5 y erfc(-y / sqrt 2) */

/*
 * rpbh_gather_rows -- the offline reordering: row k of dst = row pi(k) of src,
 * k = 0..d-1, with pi the permutation of `r` (the handle of the layer that
 * will consume the producing layer's output; OrbitQuant §2.3).
 *   src, dst   DEVICE buffers of d rows of row_bytes each, not the same buffer
 *   Use it on the producing layer's INT8 weight rows (row_bytes = K) and on
 *   its per-row scales (row_bytes = 4).  Asynchronous on `stream`.
 * Errors: RBQ_EINVAL, RBQ_ECUDA.
 */
int rpbh_gather_rows(const rbq_rpbh* r, const void* src, long long row_bytes, void* dst, void* stream);

/*
 * qlinear_int8_rotate_next -- the W8A16 layer of qlinear_int8 fused with the
 * rotation of the next layer's input, in one GEMM:
 *   y[m, j]          = scale[j] * sum_k q[j, k] * Xrot[m, k]   (the producing layer)
 *   x[m, :]          = act(y[m, :])                             (RBQ_ACT_NONE: x = y)
 *   Xrot_next[m, :]  = bf16( Pi_next x[m, :] )                  (the next layer's input,
 *                                                                as rotate_act gives it)
 * The epilogue takes each 64-column block of the accumulator (fp32), scales
 * it, applies act and the signs D of the block, the 64-point Walsh-Hadamard
 * transform and 1/8, and stores BF16 once: neither y nor x reaches memory.
 *   Xrot              device BF16 [M, K], the producing layer's rotated input
 *   Wq_next_order     device int8 [N, K]: row k = the layer's output channel
 *                     pi_next(k) (rpbh_gather_rows on the quantize_weights rows)
 *   scale_next_order  device fp32 [N], reordered the same way
 *   next              the RPBH handle of the next layer; N = its d
 *   activation        RBQ_ACT_NONE or RBQ_ACT_GELU (fp32; the normal CDF by
 *                     Abramowitz & Stegun 7.1.26, |error| <= 1.5e-7)
 *   Xrot_next         device BF16 [M, N], row-major
 * K a multiple of 64 (else RBQ_EINVAL).  Stream-ordered like qlinear_int8
 * (same workspace).
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int qlinear_int8_rotate_next(const uint16_t* Xrot, const int8_t* Wq_next_order, const float* scale_next_order,
                             int M, int K, const rbq_rpbh* next, int activation, uint16_t* Xrot_next,
                             void* stream);

/*
 * qlinear_rotate_next -- the code layer of qlinear fused with the rotation of
 * the next layer's input (OrbitQuant §6.2 on the §2.2 layer):
 *   y[m, j]          = s[m] r'[j] sum_k C_w[q_jk] C_a[p_mk]   (the producing layer)
 *   Xrot_next[m, :]  = bf16( Pi_next act(y[m, :]) )
 * as qlinear_int8_rotate_next does for the W8A16 layer; the next layer then
 * finishes its quantiser with quantize_rotated (no gather, no butterfly).
 *   a_codes, s, bits_a     the producing layer's activation codes and norms, as
 *                          for qlinear (M rows, K = its input width)
 *   w_codes_next_order     device uint8 [N, K*bits_w/8]: row k = the layer's
 *                          output channel pi_next(k) (rpbh_gather_rows on the
 *                          quantize_weights rows, row_bytes = K*bits_w/8)
 *   rnorm_next_order       device BF16 [N], reordered the same way (row_bytes 2)
 *   next                   the next layer's RPBH handle; N = its d
 *   activation             RBQ_ACT_NONE or RBQ_ACT_GELU
 *   Xrot_next              device BF16 [M, N], row-major
 * K a multiple of 128 with K*bits_a/8 a multiple of 16, N a multiple of 64
 * (else RBQ_EINVAL).  Stream-ordered like qlinear (its workspace holds both
 * operands' fp16 levels).
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int qlinear_rotate_next(const uint8_t* a_codes, const float* s, int bits_a, const uint8_t* w_codes_next_order,
                        const uint16_t* rnorm_next_order, int bits_w, int M, int K, const rbq_rpbh* next,
                        int activation, uint16_t* Xrot_next, void* stream);

/*
 * quantize_rotated -- OrbitQuant §2.2 steps 2-4 on rows that are already
 * rotated (x' = Pi_d x, e.g. from qlinear_rotate_next or rotate_act):
 * s = ||x'||, codes of x' / (s + 1e-12) in the Lloyd-Max codebook of
 * N(0, 1/d), packed as rotate_quantize_act packs them.
 *   Xrot       device BF16 [T, d] (dtype must be RBQ_BF16), row-major
 *   d          the row width (a multiple of 64; selects the codebook)
 *   bits       1..8
 *   codes_out  device uint8 [T, d*bits/8], 8-byte aligned
 *   norms_out  device fp32 [T]
 * A row whose norm is not finite is encoded as the zero vector (every code
 * 2^(bits-1)) and its norm is stored as computed.  Asynchronous on `stream`.
 * Errors: RBQ_EINVAL, RBQ_EALIGN, RBQ_ECUDA.
 */
int quantize_rotated(const void* Xrot, int dtype, int T, int d, int bits, void* codes_out, float* norms_out,
                     void* stream);

/* ---- quantised layer files ------------------------------------------------
 * The pages' "quantized model file" (INT8-convrot, section 1): the quantised
 * weights, their quantisation parameters (scale, zero point or row norms) and
 * the transform info that reproduces the rotation at inference.  One file per
 * linear layer; the transform is stored as the RPBH draw (d, h, seed, flags),
 * from which rpbh_make_ablation rebuilds pi and D exactly.  Host buffers only
 * (the caller moves them to and from the device).
 *
 * Layout (little-endian): 64-byte header -- "RBQLAYER", version u32 = 1,
 * header size u32 = 64, d, h, rpbh_flags, mode, bits, rows (i32 each),
 * seed u64, FNV-1a-64 checksum of the payload u64, zero padding -- then the
 * payload: codes, aux, zero points, back to back.
 */
#define RBQ_LAYER_LLOYDMAX    0   /* packed codes [rows, d*bits/8] + BF16 r' [rows]       */
#define RBQ_LAYER_INT8_SYM    1   /* int8 q [rows, d] + fp32 scale [rows]                  */
#define RBQ_LAYER_INT8_TENSOR 2   /* int8 q [rows, d] + fp32 scale [rows] (one value)      */
#define RBQ_LAYER_INT8_ASYM   3   /* uint8 q [rows, d] + fp32 scale + uint8 zero point [rows] */

typedef struct rbq_layer_info {
  int32_t d;           /* input width (a multiple of h)            */
  int32_t h;           /* Hadamard block size (64)                 */
  uint64_t seed;       /* RPBH seed                                */
  int32_t rpbh_flags;  /* RBQ_RPBH_NO_* of the draw                */
  int32_t mode;        /* RBQ_LAYER_*                              */
  int32_t bits;        /* code width; 8 for the INT8 modes         */
  int32_t rows;        /* output channels                          */
} rbq_layer_info;

/* rbq_layer_sizes -- payload sizes in bytes for `info` (any output may be
 * NULL).  Errors: RBQ_EINVAL for an inconsistent info. */
int rbq_layer_sizes(const rbq_layer_info* info, uint64_t* codes_bytes, uint64_t* aux_bytes, uint64_t* zp_bytes);

/* rbq_layer_write -- write a layer file.  `codes`, `aux` and (RBQ_LAYER_INT8_ASYM
 * only) `zero_point` are HOST buffers of the sizes rbq_layer_sizes gives.
 * Errors: RBQ_EINVAL, RBQ_EIO. */
int rbq_layer_write(const char* path, const rbq_layer_info* info, const void* codes, const void* aux,
                    const void* zero_point);

/* rbq_layer_read -- read a layer file's info and, when the buffer pointers are
 * not NULL, its payload into HOST buffers sized by rbq_layer_sizes(info).
 *   codes_cap, aux_cap, zp_cap  the capacities in bytes of the three buffers
 *   (zp_cap is ignored by modes without zero points).  Before anything is
 *   read into them the sizes that this file's own header gives are checked
 *   against them: a file replaced since the caller sized its buffers returns
 *   RBQ_EINVAL with the buffers untouched.
 * The checksum is verified whenever the payload is read.
 * Errors: RBQ_EINVAL, RBQ_EIO (missing, short, corrupt or foreign file). */
int rbq_layer_read(const char* path, rbq_layer_info* info, void* codes, uint64_t codes_cap, void* aux,
                   uint64_t aux_cap, void* zero_point, uint64_t zp_cap);

/* Text for a return code (static storage). */
const char* rbq_error_string(int code);

/*
 * rbq_device_error -- synchronise `stream`, then read and clear the device
 * error word of the current device.  Kernels that wait on shared-memory
 * barriers give every wait an iteration limit; when a limit runs out the
 * kernel records a non-zero word, abandons the tile and exits instead of
 * hanging.  Returns 0 when clean, RBQ_EDEVICE after such an event, RBQ_ECUDA
 * if the synchronisation itself failed.
 */
int rbq_device_error(void* stream);

/*
 * rbq_selftest_wait_limit -- launch, on `stream`, one CTA whose shared-memory
 * barriers nothing ever arrives at, so that each of the library's three
 * bounded-wait forms runs out: bit 0 of *out = a single thread's wait gave up,
 * bit 1 = a wait sharing the CTA's give-up flag gave up, bit 2 = a whole
 * warp's uniform wait gave up, bit 3 = the give-up flag was raised.  A clean
 * run leaves *out == 15 and the device error word set, so the next
 * rbq_device_error() returns RBQ_EDEVICE (and clears it).  The kernel ends by
 * itself after about a second of waiting; no other state is touched.
 * (Not a step of the method: it checks the failure handling of the kernels.)
 *
 * out: DEVICE pointer to one caller-allocated unsigned int, 4-byte aligned.
 * Errors: RBQ_EINVAL (NULL), RBQ_EALIGN, RBQ_ECUDA.
 */
int rbq_selftest_wait_limit(unsigned int* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RBQ_H */
