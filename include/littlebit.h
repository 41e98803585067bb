/*
 * littlebit.h -- C ABI of the B200 (sm_100a) LittleBit linear-layer library.
 *
 * The layer (Samsung LittleBit article, aifrontier.co.jp, section 2, the
 * "latent factorisation", "three scales" and "residual compensation" bullets)
 * approximates a weight W (d_out x d_in) as
 *     W  ~=  sum_p  diag(h_p) . U_p . diag(l_p) . V_p^T . diag(g_p)
 * with U_p in {+-1}^(d_out x s), V_p in {+-1}^(d_in x s), fp16 row scale h
 * (length d_out), column scale g (length d_in) and latent scale l (length s);
 * p runs over one path, or two when residual compensation is on, and the
 * outputs of the paths are added.  W is never formed: the forward is
 *     y = sum_p  h_p (.) ( U_p ( l_p (.) ( V_p^T ( g_p (.) x ) ) ) ).
 * Storage per layer is the effective bit width of the LittleBit-2 column
 * (physicalainews.jp, chapter 1): [s(a+b+16) + 16(a+b)] / (ab) bits per
 * weight, or [2s(a+b+16) + 32(a+b)] / (ab) with the residual path.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - Pointers named *_dev are CUDA device pointers on the current device;
 *    everything else is host memory.  The caller owns every buffer it passes.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Device work is enqueued on it and the call returns without
 *    waiting; the return value reports only what the host can check
 *    (arguments, alignment, shapes, launch errors).
 *  - The library keeps workspaces per (device, stream) -- descriptor tables
 *    and the latent-vector scratch of the forward; one each for the prefill
 *    part and each 16-row decode group of a call, and for each chunk of a
 *    host-buffer call -- allocated on first use with cudaMalloc, grown when
 *    needed and freed by littlebit_release().  Calls enqueued on the same
 *    stream are ordered; calls on different streams use different workspaces.
 *  - No entry point falls back to the CPU: without a usable CUDA device the
 *    call returns LB_ERR_CUDA.
 */
#ifndef LITTLEBIT_H
#define LITTLEBIT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  LB_OK = 0,
  LB_ERR_ARG = 1,         /* null pointer, bad enum, bad count */
  LB_ERR_ALIGN = 2,       /* a pointer is not aligned as documented */
  LB_ERR_SHAPE = 3,       /* a dimension is outside what the kernels accept */
  LB_ERR_CUDA = 4,        /* a CUDA runtime call failed (see littlebit_last_cuda_error) */
  LB_ERR_TIMEOUT = 5,     /* a bounded device wait ran out (littlebit_device_status) */
  LB_ERR_UNSUPPORTED = 6, /* a valid request this build does not implement */
  LB_ERR_RANGE = 7        /* a value left the range of the format it is held in (littlebit_device_status) */
} lb_status;

typedef enum { LB_F16 = 0, LB_BF16 = 1, LB_F32 = 2, LB_I8 = 3 } lb_dtype;

/* Which factor a packed buffer holds (see the layout below). */
typedef enum { LB_ROLE_V = 0, LB_ROLE_U = 1 } lb_role;

/*
 * Packed factor layout ("sign-plane tiles")
 * -----------------------------------------
 * A factor is viewed as a +-1 matrix F with R rows and K columns, the rows
 * being the outputs of the pass that reads it and K its contraction:
 *   LB_ROLE_V:  F[j][i] = V[i][j],  R = s,      K = d_in
 *   LB_ROLE_U:  F[o][j] = U[o][j],  R = d_out,  K = s
 * F is cut into tiles of TR x TK = 4096 elements (512 bytes):
 *   LB_ROLE_V: TR = 16,  TK = 256          LB_ROLE_U: TR = 128, TK = 32
 * R and K are zero-padded to whole tiles (padding bits are 0).  Tile (rb, kt)
 * starts at byte 512 * (rb * (Kpad / TK) + kt).  Within a tile, lane
 * L = 0..31 owns bytes 16L..16L+15 as four little-endian uint32 words
 * w_0..w_3.  With g = L / 4 and c = L % 4, bit n = 8m + q (m = 0..3,
 * q = 0..7) of w_r is the sign of element (row, k):
 *   LB_ROLE_V:  row = 16 rb + g + 8 (r % 2),         k = 256 kt + 32 q + 16 (r / 2) + 4 c + m
 *   LB_ROLE_U:  row = 128 rb + 16 q + g + 8 (r % 2), k = 32 kt + 16 (r / 2) + 4 c + m
 * and it is 1 exactly when F[row][k] < 0, i.e. sign(0) is +1.
 * Why: each lane's 16 bytes are one 128-bit load, and masking a word with
 * 0x01010101 << q leaves, byte by byte, the int8 A fragment of one
 * m16n8k32 tensor-core product for rows/columns block q (values 0 or 2^q),
 * so the decode kernels feed sign bits to the tensor cores with one logic op
 * per four signs and no unpacking.
 */

/* Bytes of a packed factor with `rows` x `cols` logical elements (R x K above). */
size_t littlebit_packed_bytes(lb_role role, int rows, int cols);

/* Effective bits per weight (LittleBit-2 column, chapter 1); host-only math. */
double littlebit_eff_bits(int d_in, int d_out, int s, int residual);

/*
 * Pack the signs of a real (or +-1) factor into the layout above: the
 * binarisation of the factors to +-1 (Samsung LittleBit article, section 2,
 * the "latent factorisation" and "Dual-SVID initialisation" bullets;
 * LittleBit-2 column, chapter 2: sign(U), sign(V)), stored one bit per sign.
 *   src_dev : factor in its natural orientation, n_long x s elements of type
 *             dt (LB_F16, LB_BF16, LB_F32 or LB_I8); element (a, j) is read at
 *             src_dev[a * stride_long + j * stride_s] (strides in elements).
 *             Role V: n_long = d_in (V is d_in x s); role U: n_long = d_out.
 *   dst_dev : littlebit_packed_bytes(role, R, K) bytes, 16-byte aligned;
 *             every byte is written (padding bits 0).
 * A NaN has no sign to keep and is packed as +1 (bit 0).
 * Errors: LB_ERR_ARG (null, bad dtype/role), LB_ERR_SHAPE (n_long or s < 1),
 * LB_ERR_ALIGN (dst not 16-byte aligned), LB_ERR_CUDA.
 */
lb_status littlebit_pack_signs(const void* src_dev, lb_dtype dt, int n_long, int s,
                               int64_t stride_long, int64_t stride_s, lb_role role,
                               void* dst_dev, void* stream);

/*
 * Inverse of littlebit_pack_signs (a test and inspection aid): the packed
 * factor at src_dev (littlebit_packed_bytes(role, R, K) bytes, 16-byte
 * aligned) back to +-1 values in its natural orientation, n_long x s int8,
 * row-major (element (a, j) at dst_dev[a * s + j]; role V: n_long = d_in,
 * role U: n_long = d_out).  Padding bits are not read.
 * Errors: LB_ERR_ARG (null, bad role), LB_ERR_SHAPE (n_long or s < 1),
 * LB_ERR_ALIGN (src not 16-byte aligned), LB_ERR_CUDA.
 */
lb_status littlebit_unpack_signs(const void* src_dev, lb_role role, int n_long, int s, int8_t* dst_dev,
                                 void* stream);

/* One path of a layer: device pointers, all owned by the caller. */
typedef struct lb_path {
  const void* V_bits;    /* packed LB_ROLE_V factor, 16-byte aligned */
  const void* U_bits;    /* packed LB_ROLE_U factor, 16-byte aligned */
  const uint16_t* h;     /* fp16 [d_out] row (output) scale, 16-byte aligned */
  const uint16_t* g;     /* fp16 [d_in]  column (input) scale, 16-byte aligned */
  const uint16_t* l;     /* fp16 [s]     latent scale */
} lb_path;

typedef struct lb_layer {
  int d_in;              /* multiple of 256, >= 256 */
  int d_out;             /* multiple of 128, >= 128 */
  int s;                 /* latent rank, 1 .. 1024 */
  int residual;          /* 0: path[0] only; 1: path[0] + path[1], same s */
  lb_path path[2];
} lb_layer;

/*
 * y = forward(x) for one layer (formula at the top of this file).
 *   x_dev : batch x d_in row-major activations, y_dev : batch x d_out.
 *   Decode (1 <= batch <= 16): x and y are fp16 (xdt = LB_F16); four kernel
 *   launches (input quantisation, latent pass, finalize, output pass), int8
 *   tensor-core products with int32 accumulation, fp32 scaling.
 *   Prefill (batch a multiple of 128, batch * d_in <= 2^30): xdt = LB_F16 or
 *   LB_BF16, y of the same type -- fp16 tcgen05 tensor-core path, see
 *   littlebit_linear_forward_many.
 *   Any other batch above 16 (fp16 only, batch * d_in <= 2^30): the leading
 *   multiple of 128 rows take the prefill path and the remaining rows the
 *   decode path in groups of at most 16 (the weights stream once per group).
 *   x_dev and y_dev must be 16-byte aligned; every other pointer as in lb_path.
 * Errors: LB_ERR_ARG, LB_ERR_ALIGN, LB_ERR_SHAPE, LB_ERR_UNSUPPORTED (a dtype
 * the batch's path does not take: bf16 below 128 rows or off a multiple of
 * 128, f32 or i8 activations), LB_ERR_CUDA.
 */
lb_status littlebit_linear_forward(const lb_layer* layer, const void* x_dev, void* y_dev,
                                   int batch, lb_dtype xdt, void* stream);

/*
 * The same forward for n independent layers (each with its own input and
 * output buffer, e.g. every linear layer of a model stack), done by the same
 * launches for the whole list (decode: the four passes; prefill: operand
 * preparation and two grouped GEMM launches per group of layers),
 * so that the weights of all layers stream from HBM back to back.  layers, xs,
 * ys are host arrays of length n.
 *
 * The library keeps a workspace per (device, stream) and remembers the last
 * call's arguments on it (the layer structs and the x and y pointers): a call
 * that repeats them enqueues kernels and events only -- no allocation, no
 * host-to-device copy -- and may therefore be captured into a CUDA graph, on
 * the same stream as an earlier eager call with the same arguments.  Kernels
 * read the pointed-to data when they run, so new contents at the same
 * addresses are picked up.
 */
lb_status littlebit_linear_forward_many(const lb_layer* layers, int n, const void* const* xs,
                                        void* const* ys, int batch, lb_dtype xdt, void* stream);

/*
 * littlebit_linear_forward_many, and in addition, on the decode path, records
 * events[i] (cudaEvent_t values passed as void*; a NULL entry is skipped) on
 * `stream` right after kernel launch i, for i < n_events <= 3: 0 = input
 * quantisation, 1 = latent pass, 2 = finalize (the output pass is last), so
 * that a caller can time each kernel with CUDA events.  The prefill path
 * records none; a batch split into groups records them in its first decode
 * group.  events may be NULL when n_events is 0.
 */
lb_status littlebit_linear_forward_many_timed(const lb_layer* layers, int n, const void* const* xs,
                                              void* const* ys, int batch, lb_dtype xdt, void* stream,
                                              void* const* events, int n_events);

/*
 * littlebit_linear_forward_many with the activations in HOST memory (no
 * counterpart in the pages; a transport wrapper around the same forward).
 *   x_host: the n layers' inputs back to back -- layer i's batch x d_in[i]
 *     row-major matrix starts at element sum_{j<i} batch * d_in[j] -- in xdt
 *     (2-byte elements).  y_host: the outputs the same way with d_out (y has
 *     x's dtype).  Both are caller-owned host memory.
 *   n_chunks (>= 1; at most min(n, 64) are used): the stack is cut into that
 *     many consecutive groups of layers of about equal bytes.  Group c's input
 *     copy, its forward and its output copy are chained by events on two
 *     library-owned copy streams and `stream`, so that copies of one group
 *     overlap the kernels of its neighbours.  Page-locked host buffers
 *     (cudaHostAlloc / cudaHostRegister) are needed for that overlap; with
 *     pageable memory the result is the same but the copies serialise.
 * Device copies of the whole stack's x and y are held per (device, stream)
 * until littlebit_release().  Both copy streams start after the work already
 * enqueued on `stream`, and `stream` continues only after the last output
 * copy, so y_host is complete once `stream` has been synchronised (the host
 * buffers must stay untouched until then).  Not for CUDA-graph capture by the
 * caller.  With page-locked buffers, the second of consecutive calls with the
 * same layers, batch, dtype, chunk count and host buffers captures the call's
 * copies and kernels as a CUDA graph, and later such calls replay it with one
 * launch; a host-buffer call with other arguments on `stream`, or
 * littlebit_release(), drops it.
 * Batch, dtype and layer rules, and errors, as littlebit_linear_forward_many;
 * LB_ERR_ARG also for NULL host pointers or n_chunks < 1.
 */
lb_status littlebit_linear_forward_many_host(const lb_layer* layers, int n, const void* x_host, void* y_host,
                                             int batch, lb_dtype xdt, int n_chunks, void* stream);

/*
 * The latent cache (Samsung LittleBit article, section 4, the KV-cache bullet:
 * because a K or V projection is factorised, the r-wide latent can be cached
 * in place of the d-wide projection).  The forward splits at t'_p = l_p (.)
 * V_p^T (g_p (.) x):
 *   littlebit_latent_forward:  x rows -> cache rows [t'_1 | t'_2]
 *   littlebit_latent_expand:   cache rows -> y = sum_p h_p (.) U_p t'_p
 * so that latent_expand(latent_forward(x)) is the layer's output up to the
 * rounding of the cache to fp16.
 * A cache row holds npaths*s fp16 values, path p at columns p*s .. p*s+s-1;
 * rows are littlebit_latent_row_elems(s, residual) elements apart (npaths*s
 * rounded up to a multiple of 8, so every row starts on 16 bytes).  For the
 * Llama-2-7B 4096x4096 projection at 0.1 BPW (s = 188, one path) a row is 192
 * values against 4096 for the projection itself: 21.3x smaller.
 */

/* Elements between cache rows of a layer of rank s (0 for an invalid s). */
int littlebit_latent_row_elems(int s, int residual);

/*
 * Cache rows of n layers' inputs: ts[i] (batch x littlebit_latent_row_elems
 * fp16, 16-byte aligned, caller-owned) receives layer i's latents of xs[i]
 * (batch x d_in, xdt).  Batch and dtype rules as littlebit_linear_forward_many
 * (decode: the input quantisation, latent pass and finalize kernels; prefill:
 * operand preparation and the first tcgen05 GEMM, whose epilogue writes the
 * rows).  Errors as littlebit_linear_forward_many.
 */
lb_status littlebit_latent_forward(const lb_layer* layers, int n, const void* const* xs, void* const* ts,
                                   int batch, lb_dtype xdt, void* stream);

/*
 * Projections rebuilt from cache rows: ys[i] (rows x d_out, ydt) = sum_p h_p
 * (.) U_p t'_p for the rows x littlebit_latent_row_elems fp16 cache rows at
 * ts[i].  rows <= 16: the cache rows are quantised to the output pass's 16-bit
 * operand (finalize kernel) and the output pass runs (ydt = LB_F16); rows a
 * multiple of 128: the rows are laid out as the second tcgen05 GEMM's operand
 * and that GEMM runs (ydt = LB_F16 or LB_BF16); other counts split as the
 * forward does.  Errors as littlebit_linear_forward_many.
 */
lb_status littlebit_latent_expand(const lb_layer* layers, int n, const void* const* ts, void* const* ys, int rows,
                                  lb_dtype ydt, void* stream);

/*
 * Initialisation of a path from real factors (the step before the forward).
 * The caller supplies the rank-s truncated SVD of the weight (any library
 * routine), split evenly: U' = U_s sqrt(S_s) (d_out x s) and V' = V_s sqrt(S_s)
 * (d_in x s), fp32 row-major on the device.
 *
 * littlebit_init_dual_svid (Samsung LittleBit article, section 2, the
 * Dual-SVID bullet: the factors' signs are the binary factors and rank-1
 * approximations of their magnitudes give the scales):
 *   U_bits_dev, V_bits_dev <- the packed signs of U', V' (sign(0) = +1; sizes
 *     littlebit_packed_bytes(LB_ROLE_U, d_out, s) and (LB_ROLE_V, s, d_in));
 *   |U'| ~ a_U b_U^T and |V'| ~ a_V b_V^T, the best rank-1 fits (top singular
 *     pairs, non-negative), found by `iters` power steps (1..1000; 32 is
 *     ample for factors of a truncated SVD);
 *   h_dev <- a_U / mean(a_U) (d_out fp16), g_dev <- a_V / mean(a_V) (d_in fp16),
 *   l_dev <- (mean(a_U) b_U) (.) (mean(a_V) b_V) (s fp16).
 * Shapes as lb_layer; every pointer 16-byte aligned (l_dev 2).  Scratch is
 * allocated and freed stream-ordered on `stream` (cudaMallocAsync).
 * For residual compensation the second path is the same initialisation of
 * the SVD of W - W_hat_1 (article section 2, residual-compensation bullet).
 *
 * littlebit_joint_itq (LittleBit-2 column, chapter 2, "solution 1"): X_dev
 * holds the stacked factors [U'; V'] (n_rows = d_out + d_in rows of s fp32);
 * `iters` (0..1000; the column's default is 50) alternations of
 * B = sign(X R) and R = the orthogonal Procrustes solution (the polar factor
 * of X^T B, by 30 Newton-Schulz steps) are run from R_dev (r_given = 1) or
 * from the identity (r_given = 0); on return R_dev holds R (s x s fp32) and
 * X_dev holds X R, i.e. U' R and V' R, whose product is U' V'^T.  Run it
 * before littlebit_init_dual_svid.  fp32 products on the CUDA cores; scratch
 * stream-ordered as above.
 * Errors: LB_ERR_ARG, LB_ERR_SHAPE, LB_ERR_ALIGN, LB_ERR_CUDA.
 */
lb_status littlebit_init_dual_svid(const float* Uf_dev, const float* Vf_dev, int d_out, int d_in, int s, int iters,
                                   void* U_bits_dev, void* V_bits_dev, uint16_t* h_dev, uint16_t* g_dev,
                                   uint16_t* l_dev, void* stream);
lb_status littlebit_joint_itq(float* X_dev, int n_rows, int s, int iters, float* R_dev, int r_given, void* stream);

/*
 * The decode forward of littlebit_linear_forward (one layer, 1 <= batch <= 16,
 * fp16 x and y) for callers that cannot let the library allocate device
 * memory: for example a process whose device memory is reserved up front by
 * its own allocator, or a latency-critical loop that cannot absorb the
 * device-wide synchronisation of cudaMalloc/cudaFree.  The pages describe no
 * such interface; it has no counterpart in them.
 *   - Allocates nothing.  Its scratch is one fixed 1 MiB device array inside
 *     the library, held by every GPU that loads the library until the process
 *     exits.  A layer whose scratch does not fit returns LB_ERR_SHAPE; per
 *     path it needs, for n = ceil(d_in/2048) input slices and r = 1 at batch 1,
 *     else 4*ceil(batch/4): n quantised input slices of 64*ceil(batch/4) +
 *     4096*r bytes, 4*ceil(n/4) * batch * 16*ceil(s/16) fp32 partial sums,
 *     and the t' bytes (about 2*r*s).
 *   - The first call on a device, with that device current, looks up the
 *     array's device address (cudaGetSymbolAddress) and zeroes its status
 *     word on `stream`; make that first call before any stream capture.
 *   - Every call shares the array and the array keeps the last call's
 *     contents; each call writes every region its kernels read before they
 *     read it.  Calls whose work overlaps on the GPU (other streams, other
 *     host threads) race on it and give wrong results: serialise them.
 *   - Device-side error bits (a bounded wait that gave up, a non-finite
 *     input) collect in the array's status word until littlebit_device_status
 *     reads and clears them.
 * Arguments, alignment and other errors as littlebit_linear_forward.
 */
lb_status littlebit_linear_forward_noalloc(const lb_layer* layer, const void* x_dev, void* y_dev,
                                           int batch, lb_dtype xdt, void* stream);

/*
 * (Host helpers below: no counterpart in the pages.)
 * Waits for `stream`, then returns in *status the device-side error bits that
 * the forward kernels enqueued on it have raised since the last call, and
 * clears them.  Bit (1 << LB_ERR_TIMEOUT) means a bounded wait for a bulk copy
 * into shared memory gave up (the outputs of that call are not valid).
 * Bit (1 << LB_ERR_RANGE) means a value could not be held in the format the
 * kernels keep it in, so the outputs of that call hold inf or NaN: an input
 * x that is inf or NaN (decode and prefill), a bf16 input beyond fp16's
 * finite range (|x| > 65504; prefill converts x to fp16), or a latent value
 * t' = l (.) t, or an fp16 output y, beyond fp16's range (prefill).
 * The word of littlebit_linear_forward_noalloc on the current device is read
 * and cleared too (its calls may be on any stream: synchronise them first).
 * *status is 0 when nothing was raised.  Errors: LB_ERR_ARG, LB_ERR_CUDA.
 */
lb_status littlebit_device_status(void* stream, unsigned int* status);

/*
 * Exercises the error path that every bounded device wait of the library
 * takes when it gives up, without any fault or hang: enqueues on `stream` one
 * kernel of one warp that polls an mbarrier that nothing completes, `polls`
 * times (each poll may suspend for up to about 1 us; 1000 polls last about a
 * millisecond), and then raises bit (1 << LB_ERR_TIMEOUT) in the status word
 * of the (device, stream) workspace.  It issues no copy, so nothing is left
 * in flight.  The next littlebit_device_status on the stream reports the bit
 * and clears it; the stream and its workspace remain usable.  Allocates the
 * workspace's status word if no forward has run on the stream yet.
 * Errors: LB_ERR_ARG (polls outside 1 .. 4194304), LB_ERR_CUDA.
 */
lb_status littlebit_check_wait_timeout(void* stream, int polls);

/* Free every workspace of every device, with its side stream and events, and
 * the device copies, copy streams and events of the host-buffer stack call
 * (call with no work in flight on any stream the library was given). */
void littlebit_release(void);

/* Human-readable name of a status code (static string). */
const char* littlebit_status_string(lb_status st);

/* Text of the last CUDA error seen by this thread (static per thread). */
const char* littlebit_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* LITTLEBIT_H */
