/*
 * fp8q -- fine-grained FP8 (E4M3) quantization and block-scaled FP8 GEMM for B200 (sm_100a).
 *
 * C ABI of libfp8q.so.  Every pointer argument marked "device" is a CUDA device
 * pointer; the caller owns all buffers (the library allocates nothing per call and
 * keeps no pointer after a call returns).  `stream` is a cudaStream_t passed as
 * void* (NULL = the legacy default stream); all work is enqueued on it, nothing
 * synchronizes the host except fp8q_get_device_error().
 *
 * Errors: arguments are validated on the host before any launch and a nonzero
 * fp8q_status is returned on the first violation; nothing aborts the process.  A
 * launch failure returns FP8Q_ERR_CUDA.  Device-side timeouts of the GEMM's bounded
 * waits are recorded in a device error word that fp8q_get_device_error() reads.
 * An empty problem (M == 0, or every group empty) is a successful no-op.
 *
 * Sources, cited by site and paragraph of the post:
 *   [Q]  the-good.kr wr_id=2169793 para 4 -- E4M3 on all tensors; the max |x| is taken
 *        online per 1x128 activation tile or 128x128 weight block and mapped to the
 *        largest FP8 value.
 *   [P2] why-be.co.kr wr_id=72410 para 1 -- scaling factors that are integral powers of 2.
 *   [K]  the-good.kr wr_id=2169793 para 1 -- per-group scaling factors along the inner
 *        dimension K, applied as dequantization on the CUDA cores; the accumulation
 *        error grows with K.
 *   [NC] pkd.ac.th webboard 78017 para 3, why-be.co.kr wr_id=57820 para 3 -- every 128
 *        K elements the tensor-core partial result is promoted: copied out, multiplied
 *        by the scaling factors and added into FP32.
 *   [MoE] why-be.co.kr wr_id=57820 para 2 (256 routed experts, 8 per token, expert size
 *        2048); pkd.ac.th webboard 78017 para 3 (decode batches per expert within 256
 *        tokens, memory-bound).
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8Q_OK = 0,
  FP8Q_ERR_NULL = 1,         /* a required pointer is NULL */
  FP8Q_ERR_SHAPE = 2,        /* negative size, K % 128 != 0, N % 128 != 0, ld too small, ... */
  FP8Q_ERR_ALIGN = 3,        /* pointer or leading dimension not 16-byte aligned as required */
  FP8Q_ERR_UNSUPPORTED = 4,  /* unknown mode / dtype, too many groups, no sm_100 device */
  FP8Q_ERR_CUDA = 5,         /* a CUDA runtime or driver call failed (launch, attribute, ...) */
  FP8Q_ERR_TIMEOUT = 6,      /* a device-side bounded wait expired (device error word only) */
  FP8Q_ERR_SCALE = 7         /* a scale is not a power of two in [2^-127, 2^127] where one is
                                required (fp8_gemm_blockscaled_ue8m0; device error word only) */
} fp8q_status;

typedef enum { FP8Q_OUT_BF16 = 0, FP8Q_OUT_FP32 = 1 } fp8q_out;

typedef enum {
  FP8Q_BSCALE_BLOCK128x128 = 0, /* B scales [N/128][K/128] row-major (weights) */
  FP8Q_BSCALE_ROW1x128 = 1      /* B scales group-major [K/128][ld_sb] (B quantized 1x128 along K) */
} fp8q_bscale;

/*
 * 1x128 activation quantization [Q], [P2].
 *
 * For every row m and group g = 0 .. K/128-1 of the bf16 matrix x:
 *   amax = max_{k<128} |x[m, 128 g + k]|
 *   s    = amax == 0 ? 1 : RN_f32(amax / 448); with pow2_scale != 0, s is raised to
 *          the smallest power of two >= s
 *   q[m, 128 g + k] = E4M3(RN_f32(x[m, 128 g + k] / s))   (nearest-even, saturate to +-448)
 *   scales[g * ld_scale + m] = s
 *
 * x_bf16  device, bf16 [M, K], row stride ldx elements (K contiguous)
 * q       device, E4M3 bytes [M, K], row stride ldq bytes
 * scales  device, fp32, group-major: [K/128][ld_scale], ld_scale >= M
 * Requires K % 128 == 0, ldx >= K and ldx % 8 == 0, ldq >= K and ldq % 8 == 0,
 * x and q 16- and 8-byte aligned, and ceil(M/64) * (K/128) <= 2^31 - 1 (one thread
 * block per 64 rows x 128 columns); otherwise FP8Q_ERR_SHAPE / FP8Q_ERR_ALIGN before
 * any launch.  Output is bit-exact with the definition above.
 */
int fp8q_quant_act_1x128(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                         int64_t ldq, float* scales, int64_t ld_scale, int pow2_scale, void* stream);

/*
 * 128x128 weight-block quantization [Q], [P2].  Same rule as above with the amax
 * taken over each 128x128 block (rows 128 nb .. +127, columns 128 g .. +127).
 *
 * w_bf16  device, bf16 [N, K], row stride ldw elements
 * q       device, E4M3 [N, K], row stride ldq bytes
 * scales  device, fp32 [N/128][K/128] row-major
 * Requires N % 128 == 0, K % 128 == 0, ldw % 8 == 0, ldq % 8 == 0, alignment as above.
 * A stack of E expert matrices [E, N, K] is one call with N' = E N.
 */
int fp8q_quant_weight_128x128(const void* w_bf16, int64_t N, int64_t K, int64_t ldw, uint8_t* q,
                              int64_t ldq, float* scales, int pow2_scale, void* stream);

/*
 * Rows and columns in one pass: the 1x128 quantization of X (exactly
 * fp8q_quant_act_1x128) and the 1x128 quantization of X^T (128x1 tiles of X, along M)
 * from one read of X [Q], [P2].  The transposed copy is what a Wgrad GEMM (dW = dY^T X)
 * consumes.  why-be.co.kr wr_id=57820 para 4 describes the HBM round trip of the
 * quantization pass; why-be.co.kr wr_id=72410 para 3 asks for support of transposed GEMM
 * operations (its text is cut off in the pages); one read serves both copies here.
 *
 * x_bf16  device, bf16 [M, K], row stride ldx elements
 * q, s    as fp8q_quant_act_1x128: E4M3 [M, K] (row stride ldq bytes), fp32 [K/128][ld_s >= M]
 * qt      device, E4M3 [K, M], row stride ldqt bytes: qt[k, m] = code of x[m, k] scaled by
 *         the amax of x[128 (m/128) .. +127, k]
 * st      device, fp32 group-major [M/128][ld_st >= K]: st[(m/128) * ld_st + k]
 * Requires M % 128 == 0, K % 128 == 0, ldx % 8 == 0, ldq % 8 == 0, ldqt % 16 == 0,
 * x and qt 16-byte aligned, q 8-byte aligned, and (M/128) * (K/128) <= 2^31 - 1 (one
 * thread block per 128x128 tile); otherwise FP8Q_ERR_SHAPE / FP8Q_ERR_ALIGN before any
 * launch.  Both outputs are bit-exact with the
 * definition (the qt / st pair equals fp8q_quant_act_1x128 applied to X^T).
 */
int fp8q_quant_act_dual(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                        int64_t ldq, float* s, int64_t ld_s, uint8_t* qt, int64_t ldqt,
                        float* st, int64_t ld_st, int pow2_scale, void* stream);

/*
 * Transpose of a matrix quantized in 128x128 blocks: qt = q^T (E4M3 [K, N], row stride
 * ldqt bytes) and st = s^T (fp32 [K/128][N/128] row-major).  A block's amax is that of
 * its transpose, so (qt, st) is exactly fp8q_quant_weight_128x128 of the transposed bf16
 * matrix -- the B operand of a Dgrad GEMM (dX = dY W, B = W^T) -- at 2 bytes of HBM
 * traffic per element instead of 3 for requantizing.
 * Requires N % 128 == 0, K % 128 == 0, ldq and ldqt multiples of 16, q and qt 16-byte
 * aligned.  Bit-exact.
 */
int fp8q_transpose_blocks(const uint8_t* q, const float* s, int64_t N, int64_t K, int64_t ldq,
                          uint8_t* qt, float* st, int64_t ldqt, void* stream);

/*
 * 1xK row quantization: one scale per row over all of K (the per-row baseline of the
 * accumulation study [K]; not part of the fine-grained path).  scales: device fp32 [M].
 * Requires K % 128 == 0 and the alignment of fp8q_quant_act_1x128.
 */
int fp8q_quant_rowwise(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                       int64_t ldq, float* scales, int pow2_scale, void* stream);

/*
 * Dense block-scaled FP8 GEMM with per-128-K promotion [K], [NC]:
 *   C[m, n] = sum_g ( sum_{k in g} A[m,k] B[n,k] ) * sA[g * ld_sa + m] * sB(n, g)
 * where the inner sum runs on the tensor cores (E4M3 x E4M3, FP32 accumulate) and the
 * scaled partials are added in FP32.  sB(n, g) = sB[(n/128) * (K/128) + g] in BLOCK mode,
 * sB[g * ld_sb + n] in ROW mode.  C = A B^T: no bias, no alpha/beta.
 *
 * A   device, E4M3 [M, K], row stride lda bytes        sA device fp32 [K/128][ld_sa], ld_sa >= M
 * B   device, E4M3 [N, K], row stride ldb bytes        sB device fp32 (layout by b_scale_mode)
 * C   device, [M, N] bf16 (FP8Q_OUT_BF16, round to nearest even) or fp32, row stride ldc elements
 * Requires K % 128 == 0, N % 128 == 0, lda/ldb >= K and multiples of 16, A/B 16-byte
 * aligned, C 16-byte aligned with ldc * sizeof(elem) a multiple of 16, ld_sa >= M,
 * ld_sb >= N (ROW mode).  M may be any size >= 0.
 */
int fp8_gemm_blockscaled(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* B,
                         const float* sB, int64_t ld_sb, int b_scale_mode, void* C, int out_dtype,
                         int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                         void* stream);

/*
 * fp8_gemm_blockscaled with bf16 output whose result is also quantized in 1x128 tiles
 * inside the GEMM's epilogue, for a following FP8 GEMM.  why-be.co.kr wr_id=57820 para 4
 * describes the HBM round trip of a separate quantization pass (read the bf16 values
 * back, write FP8 and scales) and asks for the FP8 cast to be fused with the memory
 * access; here it is fused into the producing kernel: each epilogue thread holds one row's
 * 128-column segment of the output tile, exactly one 1x128 tile.
 *
 * Results (bit-exact contract):
 *   Cb = the bf16 C of fp8_gemm_blockscaled (FP8Q_OUT_BF16) for the same arguments;
 *   (qC, sC) = fp8q_quant_act_1x128(Cb, pow2_scale): codes qC[m * ldq + n], scales
 *   sC[(n / 128) * ld_sc + m] (group-major, as the quantizer writes them).
 * C   device bf16 [M, N], row stride ldc elements, or NULL: then Cb is not stored
 * qC  device E4M3 [M, N], row stride ldq bytes        sC device fp32 [N/128][ld_sc]
 * Requires everything fp8_gemm_blockscaled requires (for C only when C is set), qC and sC
 * non-NULL, ldq >= N and a multiple of 16, qC 16-byte aligned, ld_sc >= M, sC 4-byte
 * aligned; otherwise an error before any launch.  No workspace: the last partial wave is
 * not split along K.
 */
int fp8_gemm_blockscaled_quant(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* B,
                               const float* sB, int64_t ld_sb, int b_scale_mode, void* C, int64_t ldc,
                               uint8_t* qC, int64_t ldq, float* sC, int64_t ld_sc, int pow2_scale,
                               int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb,
                               void* stream);

/*
 * fp8_gemm_blockscaled for power-of-two scales, with the scaling done inside the tensor
 * core.  why-be.co.kr wr_id=57820 para 4 and why-be.co.kr wr_id=72410 para 3 ask for
 * tensor cores that receive the scaling factors and run the MMA with group scaling; on
 * B200 that is the block-scaled MMA (tcgen05.mma kind::mxf8f6f4.block_scale), whose scale
 * factors are UE8M0 bytes, i.e. powers of two.  It multiplies every 32-element K block of
 * A and of B by its scale (exact for powers of two) and accumulates in FP32 over all of K,
 * so no per-group promotion runs on the CUDA cores.  The quantizers' pow2 option [P2]
 * produces such scales.
 *
 * Same arguments, layouts, requirements and host-side errors as fp8_gemm_blockscaled;
 * the result is the same sum, within the same acceptance band (FP32 rounding order
 * differs).  Every scale the call reads must be a power of two in [2^-127, 2^127]; any
 * other value (not a power of two, zero, negative, inf, nan) is not detectable on the
 * host: the kernel records (8 << 8) | FP8Q_ERR_SCALE in the device error word, uses 1 in
 * its place and finishes the call (C is then not the product).  Tiles of 128 x 224; no
 * workspace.
 */
int fp8_gemm_blockscaled_ue8m0(const uint8_t* A, const float* sA, int64_t ld_sa,
                               const uint8_t* B, const float* sB, int64_t ld_sb, int b_scale_mode,
                               void* C, int out_dtype, int64_t M, int64_t N, int64_t K,
                               int64_t lda, int64_t ldb, int64_t ldc, void* stream);

/*
 * fp8_gemm_grouped for power-of-two scales, scaled inside the tensor core as in
 * fp8_gemm_blockscaled_ue8m0 (one expert's rows of A against W[e] per tile, tiles of
 * 128 x 224).  Same arguments, layouts, requirements and host-side errors as
 * fp8_gemm_grouped; every scale it reads (sA for rows inside the experts, sW) must be a
 * power of two in [2^-127, 2^127], otherwise (8 << 8) | FP8Q_ERR_SCALE is recorded as for
 * fp8_gemm_blockscaled_ue8m0.
 */
int fp8_gemm_grouped_ue8m0(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* W,
                           const float* sW, void* C, int out_dtype, const int32_t* m_offsets,
                           int num_groups, int64_t max_sum_M, int64_t N, int64_t K, void* stream);

/*
 * Bytes of device workspace that fp8_gemm_blockscaled_ws can use for an M x N x K problem
 * on the current device (0 when splitting the last wave would not help).  *bytes is set
 * on success; K % 128 and N % 128 must be 0.
 */
int fp8_gemm_workspace_size(int64_t M, int64_t N, int64_t K, size_t* bytes);

/*
 * fp8_gemm_blockscaled with a caller-owned device workspace (16-byte aligned).
 *
 * When the output tiles do not fill the last wave of SMs, the tiles of that wave are split
 * along K (each chunk a whole number of 128-element groups, still promoted per group) over
 * the otherwise idle SMs; each chunk's FP32 partial tile goes to the workspace and a second
 * launch on the same stream adds the chunks in a fixed order and writes C.  Results are
 * deterministic and within the same acceptance band as the unsplit order.  With
 * workspace == NULL or workspace_bytes below fp8_gemm_workspace_size() the call computes
 * without a split (exactly fp8_gemm_blockscaled).  The workspace is scratch: its contents
 * are undefined afterwards, and calls that may run concurrently need distinct workspaces.
 */
int fp8_gemm_blockscaled_ws(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* B,
                            const float* sB, int64_t ld_sb, int b_scale_mode, void* C,
                            int out_dtype, int64_t M, int64_t N, int64_t K, int64_t lda,
                            int64_t ldb, int64_t ldc, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * fp8_gemm_blockscaled_ws for callers that cannot allocate device memory when they run the
 * GEMM -- code with a memory budget fixed in advance, allocator callbacks that must not
 * re-enter the allocator, runtimes that forbid cudaMalloc on their hot path.  The pages
 * have no counterpart to this entry point; it exists for such callers only.
 *
 * The split-K workspace is a fixed 20 MiB device array inside the library (enough for
 * every split plan on a 148-SM B200), held by every GPU that loads the library until the
 * process exits.  The call allocates and frees nothing.  The caller passes inputs and
 * outputs exactly as for fp8_gemm_blockscaled.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call before any
 *    stream capture.
 *  - Returns FP8Q_ERR_SHAPE when the problem's split would need more than 20 MiB
 *    (possible only on a GPU with more SMs), besides the errors of fp8_gemm_blockscaled.
 *  - Argument errors are those of fp8_gemm_blockscaled and are checked first.
 *  - All calls share the one array, which keeps the previous call's contents (nothing in
 *    it needs to start at zero).  Calls that can overlap on the GPU -- on different
 *    streams, or from different threads -- race on it and must be serialized by the caller.
 *  - If fp8q_get_device_error then reports a timeout, C is undefined (the reduction may
 *    have added partial tiles left by an earlier call).
 */
int fp8_gemm_blockscaled_noalloc(const uint8_t* A, const float* sA, int64_t ld_sa,
                                 const uint8_t* B, const float* sB, int64_t ld_sb,
                                 int b_scale_mode, void* C, int out_dtype, int64_t M, int64_t N,
                                 int64_t K, int64_t lda, int64_t ldb, int64_t ldc, void* stream);

/*
 * Grouped (MoE expert) block-scaled GEMM [MoE]: rows m_offsets[e] .. m_offsets[e+1]-1 of A
 * are multiplied by expert e's weights:
 *   C[m, :] = A[m, :] W[e]^T with the scaling of fp8_gemm_blockscaled (BLOCK mode).
 *
 * A          device, E4M3 [max_sum_M, K] (rows of all experts, concatenated), row stride K
 * sA         device, fp32 [K/128][ld_sa], ld_sa >= max_sum_M
 * W          device, E4M3 [num_groups, N, K] contiguous
 * sW         device, fp32 [num_groups, N/128, K/128] contiguous
 * C          device, [max_sum_M, N] bf16 or fp32, row stride N; rows outside every
 *            group are not written
 * m_offsets  device, int32 [num_groups + 1], non-decreasing, m_offsets[0] >= 0,
 *            m_offsets[num_groups] <= max_sum_M.  Read on the device: no host sync.
 * Requires 1 <= num_groups <= 1024, K % 128 == 0, N % 128 == 0, K % 16 == 0.
 */
int fp8_gemm_grouped(const uint8_t* A, const float* sA, int64_t ld_sa, const uint8_t* W,
                     const float* sW, void* C, int out_dtype, const int32_t* m_offsets,
                     int num_groups, int64_t max_sum_M, int64_t N, int64_t K, void* stream);

/*
 * No-promotion variant (accumulation study only) [K]: the whole K is accumulated in one
 * tensor-memory accumulator and per-row scales are applied once at the end:
 *   C[m, n] = ( sum_k A[m,k] B[n,k] ) * sA[m] * sB[n]      (fp32 output)
 * sA device fp32 [M], sB device fp32 [N] (from fp8q_quant_rowwise).  Shape and alignment
 * rules of fp8_gemm_blockscaled.
 */
int fp8_gemm_nopromo(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB, float* C,
                     int64_t M, int64_t N, int64_t K, int64_t lda, int64_t ldb, int64_t ldc,
                     void* stream);

/* Reads and clears the device error word (synchronizes `stream`).  Returns 0 when no
 * device-side error was recorded, else (site << 8) | fp8q_status. */
int fp8q_get_device_error(void* stream);

/* Self-test of device-side failure detection: launches a one-thread kernel whose bounded
 * wait on a barrier that nothing arrives on gives up after timeout_ns (1 ns .. 1 s) and
 * records (7 << 8) | FP8Q_ERR_TIMEOUT in the device error word.  No fault, no hang: the
 * context stays usable.  Returns FP8Q_ERR_SHAPE for an out-of-range timeout. */
int fp8q_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/* Static description of a status code. */
const char* fp8q_status_string(int status);

/* ABI version of this library (incremented on incompatible changes). */
int fp8q_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
