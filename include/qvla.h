/*
 * qvla.h -- C ABI of the B200 (sm_100a) rotated W4A4 linear layer.
 *
 *     y = s_x * s_w * ( q(R^T P^T x) . q(W P R)^T ) + b
 *
 * The method is Omega-QVLA's composite SVD.Hadamard rotation with a zigzag
 * channel permutation and per-step activation scaling.  Sources cited below:
 *  [PT]/[FR] "{Omega}-QVLA: Robust Quantization for Vision-Language-Action
 *           Models via Composite Rotation and Per-step Scaling", Portuguese
 *           and French technical summaries (gist.science), Methodology 1
 *           (composite SVD.Hadamard rotation, block implementation with the
 *           zigzag permutation) and 2 (per-step DiT activation scaling).
 *  [VN]     "Omega-QVLA: Nen VLA W4A4 tren Edge" (vnrobo.com), sections
 *           "Y tuong paper" (act_scale_table looked up per denoising step)
 *           and "Build DiT action head pack" (--use-rtn, --w-bits 4,
 *           --a-bits 4, --duquant-block-size 64).
 *  [ES]     "Omega-QVLA Reduce el Modelo ..." (aiexpert.news): a step-count
 *           mismatch or truncated table is a failure mode.
 *  [FQ]     "FoldQuantVLA: Native Low-Bit Quantization of VLA Models via
 *           Consistent Folding" (radar.vhtltd.com): dynamic per-token
 *           activation quantisation, native integer W4A4 execution.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layouts follow PyTorch Linear: W is [N][K] (out x in) row-major fp32;
 *    x is [M][ldx] row-major (bf16 or fp32); y is [M][ldy] row-major bf16.
 *  - `block` (b) is the rotation block: 32, 64, 128 or 256; K % b == 0;
 *    nb = K / b.  K <= QVLA_MAX_K.
 *  - perm[j] is the ORIGINAL input channel placed at permuted position j,
 *    so (P^T x)[j] = x[perm[j]].
 *  - rot holds the R_SVD blocks, fp32 [nb][b][b]: rot[B][i][j] is row i,
 *    column j of R_SVD of block B.  The composite block rotation is
 *    R_B = R_SVD,B . H_b with H_b the Sylvester Hadamard matrix of order b
 *    scaled by 1/sqrt(b); H is applied as a fast Walsh-Hadamard transform.
 *  - rot_tc (optional, b = 64 or 128) holds R_B itself for the tensor-core
 *    rotation: per block, R_B (computed in fp64) split into three bf16 parts
 *    hi + mid + lo (each the bf16 rounding of what the previous parts leave),
 *    each part stored as R_B^T (row j = output channel, its b inputs along
 *    the row) in the 128-byte-swizzled K-major shared-memory image of the
 *    tensor cores: 64-element K chunks of b rows x 128 bytes, the 16-byte
 *    pieces of row j XOR-permuted by (j & 7).  uint16 bf16 bits,
 *    [nb][3][b/64][b][64]; 6*K*b bytes.
 *  - Packed 4-bit codes: byte j of a row holds code 2j in its low nibble and
 *    code 2j+1 in its high nibble, 4-bit two's complement.  Weight codes lie
 *    in [-7, 7], activation codes in [-8, 7].
 *  - Rounding: the division that decides a code is an IEEE fp32 division of
 *    fp32 operands, rounded to nearest with ties to even; a zero scale gives
 *    all-zero codes.
 *  - Memory: the caller allocates every buffer.  Pointers documented as
 *    "device" must be device memory of the current CUDA device; "host"
 *    pointers are ordinary host memory.  No entry point keeps a pointer
 *    after it returns (kernels still in flight read them).
 *  - Streams: work is enqueued on `stream` (0 = legacy default stream) and
 *    runs asynchronously unless an entry point says otherwise.  The return
 *    status covers argument validation and launch errors only; errors found
 *    by a kernel while it runs set bits of the device error word, read with
 *    qvla_read_error_word().
 *  - Alignment: every device pointer must be 16-byte aligned and every row
 *    pitch a multiple of 16 bytes, or QVLA_ERR_ALIGN is returned.
 *  - Nothing is done and QVLA_OK is returned when M == 0.
 */
#ifndef QVLA_H_
#define QVLA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QVLA_ABI_VERSION 2
#define QVLA_MAX_K 32768

typedef enum {
  QVLA_OK = 0,
  QVLA_ERR_ARG = 1,          /* null pointer or invalid enum value            */
  QVLA_ERR_SHAPE = 2,        /* sizes outside the supported set               */
  QVLA_ERR_ALIGN = 3,        /* pointer or pitch not 16-byte aligned          */
  QVLA_ERR_STEP_RANGE = 4,   /* denoising step or layer outside the table     */
  QVLA_ERR_UNSUPPORTED = 5,  /* device is not sm_100 or feature unavailable   */
  QVLA_ERR_CUDA = 6,         /* a CUDA runtime call or launch failed          */
  QVLA_ERR_DEVICE_FLAG = 7,  /* the device error word was non-zero            */
  QVLA_ERR_WORKSPACE = 8     /* workspace missing or too small                */
} qvla_status;

typedef enum { QVLA_DTYPE_F32 = 0, QVLA_DTYPE_BF16 = 1 } qvla_dtype;

/* Activation scale selection ([PT]/[FR] Methodology 2; [FQ]):
 *   DYNAMIC: s_x[m] = fp32(max_k |x'[m,k]| / 7), per token.
 *   TABLE:   s_x[m] = table[step][layer] for every token (the per-step
 *            activation scale table of the DiT action head).            */
typedef enum { QVLA_SCALE_DYNAMIC = 0, QVLA_SCALE_TABLE = 1 } qvla_scale_mode;

/* Bits of the device error word. */
#define QVLA_DEVERR_STEP_RANGE 0x1u   /* device step index outside [0, T)    */
#define QVLA_DEVERR_TIMEOUT 0x2u      /* a bounded wait in a kernel expired  */
#define QVLA_DEVERR_TMEM 0x4u         /* tensor-memory allocation failed     */

/* One packed linear: what qvla_pack_weights() produces.  All pointers are
 * device pointers owned by the caller.                                     */
typedef struct {
  int32_t N, K, block;
  const int32_t* perm;      /* [K]  zigzag permutation                      */
  const float* rot;         /* [nb][b][b] R_SVD blocks, or NULL: R_SVD = I  */
                            /* (Hadamard-only rotation, R_B = H_b)           */
  const uint16_t* rot_tc;   /* tensor-core images of R_B, or NULL (with rot */
                            /* NULL: the image of R_B = H_b)                 */
  const uint8_t* wq;        /* [N][K/2] packed weight codes                 */
  const float* w_scale;     /* [N]  s_w                                      */
  const float* bias;        /* [N]  or NULL                                  */
} qvla_packed_linear;

const char* qvla_status_str(qvla_status s);
int qvla_abi_version(void);
/* SHA-256 (64 hex digits) of the sources this library was built from, as
 * the build computed it; "unstamped" for a build that set none.            */
const char* qvla_source_hash(void);

/* Reads the current device's error word into *out and, if clear != 0, resets
 * it to 0.  Synchronises the device.  Returns QVLA_ERR_CUDA on a CUDA error. */
qvla_status qvla_read_error_word(uint32_t* out, int clear);

/* Self-test of the kernels' failure path (no page counterpart: it checks this
 * library's promise that a kernel never hangs).  Launches one warp that holds
 * tensor memory and waits, with the same bounded wait every kernel here uses,
 * on a barrier nothing arrives on; after limit_ns nanoseconds it gives up,
 * sets QVLA_DEVERR_TIMEOUT in the error word, frees its tensor memory and
 * returns.  The context stays usable.  limit_ns in [1e3, 1e7], else
 * QVLA_ERR_ARG.  Asynchronous on `stream`; read the outcome with
 * qvla_read_error_word().                                                   */
qvla_status qvla_selftest_wait_timeout(uint64_t limit_ns, cudaStream_t stream);

/* Byte sizes of the buffers a packed linear needs:
 *   *wq_bytes     = N * K / 2
 *   *rot_bytes    = 4 * K * block
 *   *rot_tc_bytes = 6 * K * block for block 64 or 128, else 0 (no image)
 *   *ws_bytes     = workspace of qvla_pack_weights().  Any output may be NULL. */
qvla_status qvla_packed_sizes(int N, int K, int block, size_t* wq_bytes, size_t* rot_bytes,
                              size_t* rot_tc_bytes, size_t* ws_bytes);

/* ---------------------------------------------------------------------------
 * Offline pack ([PT]/[FR] Methodology 1: zigzag permutation by weight-column
 * norm, per-block R_SVD, normalised Hadamard, R = R_SVD . H; [VN] "Build DiT
 * action head pack": RTN, 4-bit weights, block 64).
 *
 * W        device fp32 [N][K].
 * perm_in  host int32 [K] or NULL.  NULL: the zigzag permutation is computed
 *          (column L2 norms in fp64 on the device, sorted descending with
 *          ties to the lower index, dealt to blocks in snake order).
 * rsvd_in  host fp64 [nb][b][b] or NULL.  NULL: each
 *          block's Gram matrix A_B^T A_B is formed in fp64 on the device, its
 *          eigenvectors are found on the host (cyclic Jacobi, fp64), ordered
 *          by descending eigenvalue with the largest-magnitude entry of each
 *          made positive.
 * Outputs (device): perm_out [K], rot_out [nb][b][b] fp32, rot_tc_out (may be
 *          NULL; ignored unless block is 64 or 128), wq_out [N][K/2],
 *          w_scale_out [N].  W' = W P R is formed in fp64 and
 *          rounded once to fp32 before RTN.
 * workspace device, >= ws_bytes from qvla_packed_sizes().
 * Blocks the calling thread: the stream is synchronised twice (after the
 * norms and after the Gram matrices) for the host-side sort and eigensolve.
 * ------------------------------------------------------------------------- */
qvla_status qvla_pack_weights(const float* W, int N, int K, int block, const int32_t* perm_in,
                              const double* rsvd_in, int32_t* perm_out, float* rot_out,
                              uint16_t* rot_tc_out, uint8_t* wq_out, float* w_scale_out,
                              void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Offline pack of the Hadamard-only variant: R_SVD = I for every block, so
 * R_B = H_b ("FoldQuantVLA" page: Hadamard rotation of weights and
 * activations; the composite-rotation ablation of "{Omega}-QVLA"
 * Methodology 1, SVD factor removed).  The zigzag permutation is kept:
 * perm_in host int32 [K] or NULL (computed as in qvla_pack_weights()).
 * Outputs (device): perm_out [K], rot_tc_out (optional, NULL to skip: the
 * tensor-core image of R_B = H_b for blocks 64 / 128, rot_tc_bytes of
 * qvla_packed_sizes()), wq_out [N][K/2], w_scale_out [N]; W' = W P H is
 * formed in fp64 and rounded once to fp32 before RTN.  The packed linear
 * built from these has rot = NULL; with the image, bf16 activations take the
 * tensor-core rotation, otherwise the fast Walsh-Hadamard transform alone.
 * workspace device, >= ws_bytes from qvla_packed_sizes().  Blocks the calling
 * thread (one synchronisation for the host-side sort, one at the end).
 * ------------------------------------------------------------------------- */
qvla_status qvla_pack_weights_hadamard(const float* W, int N, int K, int block,
                                       const int32_t* perm_in, int32_t* perm_out,
                                       uint16_t* rot_tc_out, uint8_t* wq_out,
                                       float* w_scale_out, void* workspace, size_t ws_bytes,
                                       cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * W8A8 variant ("FoldQuantVLA" page: attention-output and FFN-down
 * projections kept at W8A8, native integer execution).  The same zigzag
 * permutation and composite rotation as qvla_pack_weights(); weights
 * quantised symmetric per output channel to 8 bits: s_w[n] = fp32(max_k
 * |W'[n,k]| / 127), q = clamp(rint(W'/s_w), -127, 127).
 * Outputs (device): perm_out [K], rot_out [nb][b][b] fp32, wq_out [N][K]
 * int8 (one code per byte: N * K bytes, not the N * K / 2 of
 * qvla_packed_sizes()), w_scale_out [N], and optionally rot_tc_out (the
 * tensor-core image of R_B as in qvla_pack_weights(), NULL to skip; with it
 * the activation rotation of qvla_rotate_quant_act_a8() runs on the tensor
 * cores).  Its wq must only be given to qvla_w8a8_gemm() /
 * qvla_w8a8_gemm_s32().  Other arguments and the blocking behaviour as
 * qvla_pack_weights().
 * ------------------------------------------------------------------------- */
qvla_status qvla_pack_weights_w8(const float* W, int N, int K, int block, const int32_t* perm_in,
                                 const double* rsvd_in, int32_t* perm_out, float* rot_out,
                                 uint16_t* rot_tc_out, uint8_t* wq_out, float* w_scale_out,
                                 void* workspace, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * GPTQ rounding of rotated weights ("Omega-QVLA: Nen VLA W4A4 tren Edge",
 * "Build LLM pack": the LLM pack's 4-bit weights come from GPTQ on the
 * composite-rotated weights, block 128, damping 0.05).  Host only, fp64.
 *   H  = X'^T X' of the rotated calibration rows X' (K x K);
 *   dead inputs (H[i][i] == 0) get H[i][i] = 1 and a zero weight column;
 *   U  = upper Cholesky factor of (H + damp * mean(diag H) * I)^-1;
 *   per row: s = fp32(max_k |W'[n,k]| / 7) (the RTN scale); for j = 0..K-1:
 *     q_j = clamp(rint(w_j / s), -7, 7); e = (w_j - q_j s) / U[j][j];
 *     w_k -= e U[j][k] for k > j.
 * The pages' block size only groups the lazy updates; it does not change the
 * result, and here every update is applied as its column is done.
 *
 * qvla_gptq_quantize_host: Wr host fp32 [N][K] (rotated weights W' = W P R);
 * H host fp64 [K][K] (symmetric) or NULL when u_in is given; u_in host fp64
 * [K][K] upper factor U (used as is; then H and damp are ignored) or NULL;
 * q_out host int8 [N][K] codes in [-7, 7]; s_out host fp32 [N].  K <= 4096
 * (QVLA_ERR_SHAPE otherwise: the work is K x K fp64 on the host);
 * QVLA_ERR_ARG if a factorisation fails.  Synchronous, multithreaded.
 * ------------------------------------------------------------------------- */
qvla_status qvla_gptq_quantize_host(const float* Wr, int N, int K, const double* H, double damp,
                                    const double* u_in, int8_t* q_out, float* s_out);

/* H = X'^T X' in fp64 (K x K, row-major, symmetric) of the rotated
 * calibration rows xr host fp32 [T][K], into H_out host fp64 [K][K] (the
 * Hessian the GPTQ entry points factorise).  K <= 4096.  Synchronous.       */
qvla_status qvla_gptq_hessian_host(const float* xr, int T, int K, double* H_out);

/* Offline pack with GPTQ weights: as qvla_pack_weights() (same perm_in,
 * rsvd_in, outputs, workspace and blocking behaviour), but wq_out and
 * w_scale_out hold the GPTQ codes of W' instead of the RTN codes.  The
 * calibration rows x_cal (device, xdt F32 or BF16, [T][K] dense) are
 * rotated on the device with P and R (as qvla_rotate_act_f32(), into
 * cal_workspace, >= T * K * 4 bytes) and H is formed on the host in fp64.
 * u_in host fp64 [K][K] or NULL: a given U skips the calibration (x_cal,
 * T and cal_workspace may then be NULL / 0).  damp >= 0.  K <= 4096.        */
qvla_status qvla_pack_weights_gptq(const float* W, int N, int K, int block, const void* x_cal,
                                   qvla_dtype xdt, int T, double damp, const int32_t* perm_in,
                                   const double* rsvd_in, const double* u_in, int32_t* perm_out,
                                   float* rot_out, uint16_t* rot_tc_out, uint8_t* wq_out,
                                   float* w_scale_out, void* workspace, size_t ws_bytes,
                                   void* cal_workspace, size_t cal_ws_bytes, cudaStream_t stream);

/* W8A8 activations: the rotation of qvla_rotate_act_f32() into `workspace`
 * (fp32 [M][K] at its start, M * K * 4 bytes), then per-token dynamic 8-bit
 * RTN: s_x[m] = fp32(max_k |x'[m,k]| / 127), q = clamp(rint(x'/s_x), -128,
 * 127), one int8 code per byte.  When the workspace holds M * K * 6 bytes
 * (qvla_rotate_quant_a8_workspace_bytes) the last M * K * 2 take the
 * permuted copy of x that the tensor-core rotation reads through TMA (bf16
 * input and a linear that carries a tensor-core image, block 64 / 128; a
 * pack without the image rotates on the CUDA cores and leaves that part
 * unused); with M * K * 4 the rotation gathers instead (same result).  x, xdt, ldx, L as in qvla_rotate_quant_act().  Outputs
 * (device): xq8 [M][K] int8, s_x [M] fp32.  Asynchronous (two or three
 * launches).                                                               */
qvla_status qvla_rotate_quant_act_a8(const void* x, qvla_dtype xdt, int M, int ldx,
                                     const qvla_packed_linear* L, int8_t* xq8, float* s_x,
                                     void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Scratch of qvla_rotate_quant_act_a8() for its fastest route: M * K * 6
 * bytes (M * K * 4 is the minimum).                                         */
qvla_status qvla_rotate_quant_a8_workspace_bytes(int M, int K, size_t* bytes);

/* W8A8 GEMM: acc[m,n] = sum_k xq8[m,k] wq[n,k] (int8 x int8 -> int32, exact
 * for K <= QVLA_MAX_K), y = bf16(fp32(s_x[m] s_w[n]) * acc + b[n]) — the W4A4
 * epilogue.  xq8 device [M][K] int8 from qvla_rotate_quant_act_a8(); L from
 * qvla_pack_weights_w8() (wq [N][K] int8); y device bf16 [M][ldy] (ldy >= N,
 * ldy * 2 a multiple of 16).  The int8 codes go to the tensor cores as they
 * are (no unpack).  Asynchronous.                                          */
qvla_status qvla_w8a8_gemm(const int8_t* xq8, const float* s_x, int M,
                           const qvla_packed_linear* L, void* y, int ldy, cudaStream_t stream);

/* The int32 accumulators of qvla_w8a8_gemm() into acc [M][N] (tests).       */
qvla_status qvla_w8a8_gemm_s32(const int8_t* xq8, int M, const qvla_packed_linear* L,
                               int32_t* acc, cudaStream_t stream);

/* Device step of the pack: W'_f32 = fp32(W P R), computed in fp64 from fp64
 * R_SVD blocks.  W device fp32 [N][K]; perm device [K]; rsvd64 device fp64
 * [nb][b][b]; Wr_out device fp32 [N][K].  Asynchronous.                    */
qvla_status qvla_rotate_weights_f32(const float* W, int N, int K, int block, const int32_t* perm,
                                    const double* rsvd64, float* Wr_out, cudaStream_t stream);

/* Device step of the pack: RTN + nibble packing of fp32 rotated weights.
 * s_w[n] = fp32(max_k |W'[n,k]| / 7); q = clamp(rint(W'/s_w), -7, 7).
 * Asynchronous.                                                            */
qvla_status qvla_quant_pack_weights_f32(const float* Wr, int N, int K, uint8_t* wq_out,
                                        float* w_scale_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Run-time activation rotate + quantise: one fused kernel per token tile.
 * For each token row m: gather x[m, perm[j]], apply R_SVD,B^T per block,
 * then the fast Walsh-Hadamard transform (scaled by 1/sqrt(b)), select the
 * scale (DYNAMIC or TABLE), round to 4-bit codes and nibble-pack them.
 *
 * x       device, [M][ldx] of `xdt` (ldx >= K, in elements).
 * L       host pointer to a packed linear (device pointers inside); only
 *         perm, rot, rot_tc, K and block are read.  rot = NULL (Hadamard-only
 *         linear): the gathered block goes straight to the fast Walsh-Hadamard
 *         transform, no R_SVD product.  With bf16 input and a
 *         rot_tc image the rotation runs on the tensor cores as one dense
 *         product with R_B = R_SVD,B . H_b (three bf16 parts, fp32
 *         accumulation in tensor memory); otherwise on the CUDA cores as the
 *         R_SVD product followed by the fast Walsh-Hadamard transform
 *         (fp32 input at block 64 in TABLE mode: one dense product with the
 *         fp32 sum of the image's three parts).
 * table   device fp32 [T][Lcount], required for TABLE mode.
 * step_dev device int32 or NULL.  If non-NULL the step is read on the device
 *         (so one captured graph serves every denoising step); a step outside
 *         [0, T) sets QVLA_DEVERR_STEP_RANGE and the kernel writes all-zero
 *         codes and s_x = 0 (y becomes the bias) rather than reading outside
 *         the table ([ES]).  If NULL, `step_host` is used and checked on the
 *         host (QVLA_ERR_STEP_RANGE).
 * layer   column of the table; 0 <= layer < Lcount (checked on the host).
 * workspace optional device scratch (see qvla_rotate_quant_workspace_bytes).
 * Outputs (device): xq [M][K/2] packed codes, s_x [M] fp32.
 * ------------------------------------------------------------------------- */
qvla_status qvla_rotate_quant_act(const void* x, qvla_dtype xdt, int M, int ldx,
                                  const qvla_packed_linear* L, qvla_scale_mode mode,
                                  const float* table, int T, int Lcount, const int32_t* step_dev,
                                  int step_host, int layer, uint8_t* xq, float* s_x,
                                  void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Scratch that lets qvla_rotate_quant_act take its fastest route
 * (tensor-core rotation fed by TMA from a permuted copy of x):
 * M * K * 2 + M * (K / block) * 4 bytes when that route applies (bf16 input,
 * block 64 or 128, M > 0), else 0.  The first M * K * 2 bytes hold the
 * permuted copy; the rest, in DYNAMIC mode, the row maxima of each CTA when
 * the two passes (maximum, then quantisation) run as two launches, which
 * spreads the blocks of wide and narrow linears evenly over the SMs.  With
 * only M * K * 2 bytes the DYNAMIC passes run in one launch, the maximum
 * reduced over a thread-block cluster; without scratch (workspace NULL or
 * smaller) the call still works, gathering the permuted inputs directly.
 * All routes give the same codes and scales.  The scratch is only used
 * while the call's kernels run; reusing it for another call on the same
 * stream is safe.                                                          */
qvla_status qvla_rotate_quant_workspace_bytes(int M, int K, int block, qvla_dtype xdt,
                                              size_t* bytes);

/* qvla_rotate_quant_act without any allocation by the caller or the library.
 * (No counterpart in the paper: this is a deployment convenience.)
 * For callers that cannot allocate device memory when they run a layer --
 * an inference loop that must not call cudaMalloc once it is running (a
 * robot control loop with a hard cycle budget, code that is being captured
 * into a CUDA graph, a host application that hands out no allocator) -- the
 * scratch the tensor-core route needs (qvla_rotate_quant_workspace_bytes)
 * lives in a fixed array inside the library, QVLA_NOALLOC_SCRATCH_BYTES bytes
 * per device, kept for as long as the library is loaded.  Arguments and
 * results are those of qvla_rotate_quant_act.
 *  - A call whose permuted copy (M * K * 2 bytes, when the tensor-core
 *    route applies) exceeds QVLA_NOALLOC_SCRATCH_BYTES returns
 *    QVLA_ERR_WORKSPACE and does nothing.  The DYNAMIC row maxima that
 *    follow it in a full workspace are used only when they fit as well.
 *  - The first call on a device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *  - Every call on a device shares the one array: calls that may run at the
 *    same time on the GPU (different streams, no ordering) race on it.  The
 *    array keeps the last call's contents; nothing in it needs to start at
 *    zero (each call writes every byte it later reads).                    */
#define QVLA_NOALLOC_SCRATCH_BYTES (16u << 20)
qvla_status qvla_rotate_quant_act_noalloc(const void* x, qvla_dtype xdt, int M, int ldx,
                                          const qvla_packed_linear* L, qvla_scale_mode mode,
                                          const float* table, int T, int Lcount,
                                          const int32_t* step_dev, int step_host, int layer,
                                          uint8_t* xq, float* s_x, cudaStream_t stream);

/* The rotation alone, for parity checks: xr_out device fp32 [M][K] = the
 * same fp32 x' the fused kernel quantises.                                  */
qvla_status qvla_rotate_act_f32(const void* x, qvla_dtype xdt, int M, int ldx,
                                const qvla_packed_linear* L, float* xr_out, cudaStream_t stream);

/* The quantiser alone, from fp32 rotated activations xr [M][K] (device):
 * identical scale selection, rounding and packing as the fused kernel.     */
qvla_status qvla_quant_act_f32(const float* xr, int M, int K, qvla_scale_mode mode,
                               const float* table, int T, int Lcount, const int32_t* step_dev,
                               int step_host, int layer, uint8_t* xq, float* s_x,
                               cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * W4A4 GEMM with fused dequantisation:
 *   acc[m,n] = sum_k q_x[m,k] q_w[n,k]            (exact, int32)
 *   y[m,n]   = bf16( fp32(s_x[m] * s_w[n]) * fp32(acc) + b[n] )
 * The int4 weight codes are unpacked to 8-bit values in tensor memory and
 * multiplied on the tcgen05 tensor cores (kind::i8, A operand from tensor
 * memory, int32 accumulators in tensor memory); the activation codes are
 * unpacked in shared memory (or read as the int8 image, see
 * qvla_linear_problem.xq8).  Each code q enters as the int8 value 16*q (a
 * nibble moved into the high half of its byte), so the tensor cores
 * accumulate 256*acc exactly (|256*acc| <= 256*64*K < 2^31 for
 * K <= QVLA_MAX_K) and the epilogue shifts it back.
 * One persistent CTA per SM walks a list of 128-channel x (16..128)-token
 * tiles that the host deals out longest first; no workspace.  For token
 * tiles of at most 64, a tile much longer than the average list may be split
 * over K between the two CTAs of a cluster, the second sending its int32
 * partial through distributed shared memory (the sum is exact either way).
 * xq device [M][K/2]; s_x device [M]; y device bf16 [M][ldy].
 * split_k: 0, 1, 2, 4, 8 or 16, at most ceil(K / 256); accepted for source
 * compatibility and otherwise ignored (the tile schedule balances the work;
 * results do not depend on it).
 * N may be any positive size up to 2^22 and M up to 2^20 (QVLA_ERR_CUDA
 * beyond); ragged M, N and K tails are zero-filled.                          */
qvla_status qvla_w4a4_gemm(const uint8_t* xq, const float* s_x, int M,
                           const qvla_packed_linear* L, void* y, int ldy, int split_k,
                           cudaStream_t stream);

/* Same GEMM, writing the raw int32 accumulators acc [M][N] (device) instead
 * of y, for bit-exact parity checks.                                        */
qvla_status qvla_w4a4_gemm_s32(const uint8_t* xq, int M, const qvla_packed_linear* L,
                               int32_t* acc, int split_k, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Batched calls: several INDEPENDENT linears (each with its own packed
 * weights, input, codes and output; e.g. the gate and up projections of an
 * MLP, q/k/v, or the linears of a denoising step whose inputs are already
 * known) run in as few launches as possible instead of one launch each.
 * Linears are grouped by kernel configuration (rotation block, token tile,
 * input type, scale mode); each launch takes up to 16 of them.  Results are
 * identical to calling the single-linear entry points one by one.  No two
 * problems may share an output buffer, and their workspaces must not
 * overlap (the problems of one call run at the same time): the batched
 * rotate-quantise returns QVLA_ERR_ARG when two non-NULL workspace ranges
 * [workspace, workspace + ws_bytes) intersect.
 * ------------------------------------------------------------------------- */
typedef struct {
  const qvla_packed_linear* L;   /* host pointer to the packed linear          */
  const void* x;                 /* device [M][ldx] activations (rotate-quant) */
  int32_t xdt;                   /* qvla_dtype                                  */
  int32_t M, ldx;
  int32_t mode;                  /* qvla_scale_mode                             */
  const float* table;            /* device [T][Lcount] for TABLE mode           */
  int32_t T, Lcount;
  const int32_t* step_dev;       /* device step index or NULL (use step_host)   */
  int32_t step_host, layer;
  uint8_t* xq;                   /* device [M][K/2] codes: output, then input   */
  float* s_x;                    /* device [M] scales: output, then input       */
  void* y;                       /* device bf16 [M][ldy] GEMM output            */
  int32_t ldy;
  void* workspace;               /* optional rotate-quant scratch, or NULL      */
  size_t ws_bytes;               /* (qvla_rotate_quant_workspace_bytes)         */
  int8_t* xq8;                   /* optional device [M][K] int8 image of the    */
                                 /* codes (see below), or NULL                  */
} qvla_linear_problem;

/* The int8 image of the activation codes (xq8), the GEMM's B operand as the
 * tensor cores take it: byte k of a row is 16 * q[j] with, inside every
 * aligned group of 32 codes, the 16 even-indexed codes first and then the 16
 * odd-indexed ones (k = 32g + i holds code 32g + 2i for i < 16 and code
 * 32g + 2(i - 16) + 1 otherwise).  It is a fixed rearrangement of xq: each
 * packed byte's low nibble moves to the high half of one image byte and its
 * high nibble to another.  When a problem gives xq8, the batched
 * rotate-quantise writes it next to xq and s_x, and the batched GEMM reads
 * its activations from it (one TMA box straight into the MMA layout) instead
 * of unpacking xq; the results are identical.  Row pitch K, 16-byte aligned. */

/* qvla_rotate_quant_act for every problem (reads x, writes xq and s_x). */
qvla_status qvla_rotate_quant_act_batched(const qvla_linear_problem* probs, int n,
                                          cudaStream_t stream);

/* qvla_w4a4_gemm for every problem (reads xq and s_x, writes y); split_k as
 * for qvla_w4a4_gemm, one factor shared by all problems of a launch.        */
qvla_status qvla_w4a4_gemm_batched(const qvla_linear_problem* probs, int n, int split_k,
                                   cudaStream_t stream);

/* The W8A8 linears of a step, batched the same way (the variant the pages keep
 * at 8 bits for the attention-output and FFN-down projections).  For these
 * two entry points each problem's xq8 holds the 8-bit codes themselves
 * (device int8 [M][K], one code per byte: q, not 16 * q), L is a pack from
 * qvla_pack_weights_w8(), and xq is not used.
 * qvla_rotate_quant_act_a8_batched: qvla_rotate_quant_act_a8() for every
 * problem (reads x, writes xq8 and s_x); each problem's workspace /
 * ws_bytes is its scratch as in qvla_rotate_quant_act_a8() (at least
 * M * K * 4 bytes, else QVLA_ERR_WORKSPACE; M * K * 6 for the tensor-core
 * route), 16-byte aligned, and no two workspaces may overlap (QVLA_ERR_ARG).
 * mode, table and step fields are ignored (8-bit activations take the
 * per-token dynamic scale).  Two launches for all problems (the rotations,
 * then the row quantisation), plus the permuted copy on the tensor-core route.
 * qvla_w8a8_gemm_batched: qvla_w8a8_gemm() for every problem (reads xq8,
 * s_x, writes y), one launch per token tile for up to 16 linears.
 * Results are identical to the single-linear calls.  Asynchronous.         */
qvla_status qvla_rotate_quant_act_a8_batched(const qvla_linear_problem* probs, int n,
                                             cudaStream_t stream);
qvla_status qvla_w8a8_gemm_batched(const qvla_linear_problem* probs, int n, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* QVLA_H_ */
