/*
 * tq.h -- C ABI of the B200 (sm_100a) TurboQuant hot path.
 *
 * TurboQuant is an online, data-oblivious vector quantizer.  Pages cited below:
 *   [ttakun]  "KV缓存52GB瞬间爆内存？TurboQuant随机旋转+标量量化如何把LLM长上下文推理成本
 *             砍到1/16且失真逼近理论极限" (ttakun.com/news/45354)
 *   [tmdm]    "谷歌悄悄扔下一颗“性能核弹”：KV缓存压缩6倍，推理提速8倍，还不用重训模型"
 *             (tmdm.cn/turboquant-kv-compression)
 *   [admirer] m.admirer.cn report on "TurboQuant: Online Vector Quantization with
 *             Near-optimal Distortion Rate" (arXiv 2504.19874)
 *   [tq.net]  turboquant.net/zh, "TurboQuant 最近的进展和外溢影响"
 *
 * Conventions shared by every call
 * --------------------------------
 * - Return value: TQ_OK (0) or one of the TQ_E* codes below.  On error the
 *   call has launched nothing; tq_last_error() returns a message for the
 *   calling thread.
 * - Device pointers ("dev") are caller-owned device memory on the handle's
 *   device; the library never allocates, frees or retains them.  Host
 *   pointers ("host") are read or written before the call returns.
 * - Every device call is asynchronous on `stream` (a cudaStream_t, NULL = the
 *   legacy default stream) and does not synchronise.  Outputs are complete
 *   when the stream reaches the call.
 * - Alignment: every device pointer must be 16-byte aligned (TQ_EALIGN).
 * - A handle holds only constants (rotation, projection, codebook) uploaded
 *   by tq_create to the device that was current at that time.  Concurrent
 *   calls on one handle from several streams are safe; destroying a handle
 *   while work that uses it is in flight is not.
 * - A kernel that meets a condition it cannot finish under (a pipeline wait
 *   that runs past its time limit, a shared-memory window that is not where
 *   tq_create measured it) leaves early and sets a bit in the handle's device
 *   status word; the call has already returned TQ_OK by then, and that call's
 *   outputs are incomplete.  Callers that must know poll tq_device_status
 *   after their stream has reached the calls in question.
 *
 * Packed code layout (the pages say only that 32-bit coordinates become 2- or
 * 4-bit integers, [ttakun, "为什么随机旋转是整个算法的底层杠杆"]).  A vector's d rotated
 * coordinates form G = ceil(d/32) groups of 32 (coordinates past d are zero);
 * group g owns the b consecutive uint32 words g*b .. g*b+b-1, so one vector
 * takes TQ_CODE_WORDS(b, d) = G*b words.  Inside a group, for local coordinate i:
 *   b = 1: word 0 bit i = idx_i
 *   b = 2: word k bits 2j..2j+1 = idx_{16k+j}          (k < 2, j < 16)
 *   b = 3: word k bits 4j..4j+2 = idx_{8k+j}           (k < 3, j < 8)
 *          word k bit  4j+3     = bit k of idx_{24+j}
 *   b = 4: word k bits 4j..4j+3 = idx_{8k+j}           (k < 4, j < 8)
 * QJL sign bits use the b = 1 layout (bit set <=> (S r)_i >= 0).
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define TQ_OK 0
#define TQ_EINVAL 1        /* NULL pointer, negative size, inconsistent shapes */
#define TQ_EUNSUPPORTED 2  /* b, d, dtype or variant outside the supported set */
#define TQ_EALIGN 3        /* a device pointer is not 16-byte aligned */
#define TQ_ECUDA 4         /* a CUDA runtime call or launch failed (see tq_last_error) */
#define TQ_ENOMEM 5        /* tq_create could not allocate the handle's constants */
#define TQ_EWORKSPACE 6    /* the workspace passed is smaller than required */

/* element types */
#define TQ_F32 0
#define TQ_BF16 1
#define TQ_F16 2  /* storage of residual norms only (tq_quant_paged, tq_attn_decode_paged) */

/* variants */
#define TQ_MSE 0  /* TurboQuant_mse: b bits per coordinate */
#define TQ_PROD 1 /* TurboQuant_prod: (b-1)-bit mse + 1-bit QJL of the residual */

#define TQ_MAX_DIM 4096
#define TQ_CODE_WORDS(b, d) ((((d) + 31) / 32) * (b))
#define TQ_SIGN_WORDS(d) (((d) + 31) / 32)

typedef struct tq_ctx* tq_handle;

/* ---------------------------------------------------------------- host setup */

/*
 * tq_make_codebook -- Lloyd-Max scalar quantizer for one rotated coordinate.
 * [ttakun, "为什么随机旋转是整个算法的底层杠杆"]: after the rotation each coordinate
 * follows a known Beta-shaped law and is quantized with a precomputed Lloyd-Max
 * quantizer; the law is f(x) = Gamma(d/2)/(sqrt(pi) Gamma((d-1)/2)) (1-x^2)^((d-3)/2)
 * on [-1, 1] [tq.net, "TurboQuant 两阶段算法", 坐标分布公式]; computed once offline
 * [tq.net, "实现步骤草图", 预计算 Lloyd-Max 质心].
 *   b           bits, 1..4
 *   d           dimension, 3..TQ_MAX_DIM
 *   centroids   host out, [2^b] ascending, float64, symmetric (c_k = -c_{2^b-1-k})
 *   thresholds  host out, [2^b - 1], midpoints of adjacent centroids (may be NULL)
 * Iterates to the float64 fixed point.  Pure host code; needs no GPU.
 * Errors: TQ_EINVAL (NULL centroids), TQ_EUNSUPPORTED (b or d out of range).
 */
TQ_API int tq_make_codebook(int b, int d, double* centroids, double* thresholds);

/*
 * tq_make_rotation -- random orthogonal rotation from a Gaussian matrix.
 * [ttakun, "为什么随机旋转是整个算法的底层杠杆"]: the rotation is obtained from the QR
 * decomposition of a random Gaussian matrix; [tq.net, "实现步骤草图", 生成随机旋转矩阵].
 *   d    dimension, 1..TQ_MAX_DIM
 *   G    host in, [d*d] row-major float64 (caller's N(0,1) draws)
 *   Pi   host out, [d*d] row-major float64: Q of G = Q R (Householder), with
 *        column j multiplied by sign(R_jj) so that R has a positive diagonal
 *        (Haar distributed).  The quantizer uses y = Pi x.
 * Pure host code.  Errors: TQ_EINVAL, TQ_EUNSUPPORTED (d), TQ_ENOMEM.
 */
TQ_API int tq_make_rotation(int d, const double* G, double* Pi);

/*
 * tq_create -- upload the constants of one quantizer instance.
 *   h          host out, the new handle
 *   d          dimension; supported: 8..TQ_MAX_DIM with d % 8 == 0
 *   b          total bits per coordinate: TQ_MSE 1..4, TQ_PROD 2..4
 *              (TQ_PROD spends b-1 bits on the mse stage and 1 on QJL)
 *   variant    TQ_MSE or TQ_PROD
 *   Pi         host in, [d*d] row-major float64 orthogonal rotation (y = Pi x)
 *   S          host in, [d*d] row-major float64 QJL projection (m = d rows);
 *              NULL for TQ_MSE.  Reading: the pages never give S's shape; the
 *              estimator's sqrt(pi/2)/d factor implies m = d.
 *   centroids  host in, [2^bm] ascending (bm = b for TQ_MSE, b-1 for TQ_PROD),
 *              or NULL to use tq_make_codebook(bm, d)
 * Allocates device memory for the constants on the current device (the only
 * allocation the library makes), launches one 32-thread kernel that reports
 * where a kernel's dynamic shared-memory window starts (the decode and logits
 * kernels address their lookup tables from it), and synchronises.  With the
 * environment variable TQ_RUNTIME_TABLE_ADDRESSES=1 the probe is skipped and
 * those kernels add the table addresses at run time (a slower instance of the
 * same arithmetic).
 * Two diagnostic settings, also read from the environment here, exist so that
 * the status word's reports can be exercised without faulting a GPU (both are
 * off unless set):
 *   TQ_DEBUG_STALL_MS=m  tq_attn_decode's kernel first waits, m ms at most, on
 *                        a barrier that nothing completes, and every other wait
 *                        of that kernel gives up after m ms: the call reports
 *                        TQ_STATUS_TIMEOUT and its output is undefined
 *   TQ_DEBUG_DYN_BASE=a  record `a` as the measured shared-window address, so
 *                        the decode (mma.sync) and logits kernels built for the
 *                        usual address report TQ_STATUS_LAYOUT and write nothing
 * and two that select between implementations of the same arithmetic:
 *   TQ_FUSED_REGISTER_LOADS=1  quantization at d <= 256 takes the kernel whose
 *                        producer threads load x themselves (the one a channel
 *                        gather always takes) instead of the TMA-staged one
 *   TQ_TCGEN05_ATTN=1    tq_attn_decode on a dense cache and the two-group
 *                        tq_attn_logits take the tcgen05 kernels instead of
 *                        the mma.sync ones (a paged cache always takes the
 *                        mma.sync decode kernel)
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ENOMEM, TQ_ECUDA.
 */
TQ_API int tq_create(tq_handle* h, int d, int b, int variant, const double* Pi, const double* S,
              const double* centroids);

/* tq_destroy -- free the handle's device constants (synchronises the device). NULL is a no-op. */
TQ_API int tq_destroy(tq_handle h);

/* tq_handle_info -- d, b, variant and bm (mse bits) of a handle; any out pointer may be NULL. */
TQ_API int tq_handle_info(tq_handle h, int* d, int* b, int* variant, int* mse_bits);

/* ---------------------------------------------------------------- hot path */

/*
 * tq_quant_mse -- TurboQuant_mse quantization of N vectors
 * ([ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: store the norm as
 * float32, rotate, quantize every coordinate independently against the
 * precomputed codebook; [tq.net, "实现步骤草图", quant 原语]).
 * n_i = ||x_i||, y = Pi x_i / n_i, idx_j = #{k : y_j >= t_k} (ties go up),
 * codes packed as described at the top of this file.  x_i = 0 gives n_i = 0
 * and the codes of y = 0.
 *   h         handle with variant TQ_MSE
 *   x         dev in, N rows of d elements of `dtype` (TQ_F32 or TQ_BF16),
 *             row i at x + i*x_stride elements; x_stride >= d, x_stride % 8 == 0
 *   N         number of vectors (0 is a no-op)
 *   codes     dev out, row i at codes + i*out_stride*TQ_CODE_WORDS(b, d)
 *   norms     dev out, float32, norms[i*out_stride]
 *   out_stride  >= 1; 1 for dense outputs (a larger stride writes every
 *             out_stride-th slot, e.g. one token slot per head of a KV cache)
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_quant_mse(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                 uint32_t* codes, float* norms, int64_t out_stride, void* stream);

/*
 * tq_dequant_mse -- x_hat_i = n_i * Pi^T c[idx_i]
 * ([ttakun, same section]: rebuild by rotating back and rescaling;
 * [tq.net, "实现步骤草图", dequant 原语]).
 *   h       handle with variant TQ_MSE (or TQ_PROD: dequantizes its mse stage)
 *   codes   dev in, [N][TQ_CODE_WORDS(bm, d)]
 *   norms   dev in, [N] float32
 *   out     dev out, [N][d] of out_dtype (TQ_F32 or TQ_BF16)
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_dequant_mse(tq_handle h, const uint32_t* codes, const float* norms, int64_t N, void* out,
                   int out_dtype, void* stream);

/*
 * tq_quant_prod -- TurboQuant_prod quantization
 * ([ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: (b-1)-bit mse gives
 * x_hat and the residual r, then 1-bit QJL of r; [tmdm, "双剑合璧：PolarQuant + QJL",
 * ✦ QJL]; [admirer, "第二步：1 bit 算力帶來的「神級校準」"]).
 * Computes the mse stage as tq_quant_mse with bm = b-1 bits, then in the
 * rotated frame u = y - c[idx] (so r = n Pi^T u), sign bits of (S r)_j =
 * n (S Pi^T u)_j (bit set <=> >= 0), and rn = ||r|| = n ||u||.
 *   x, N, x_stride, out_stride   as tq_quant_mse
 *   codes    dev out, [N][TQ_CODE_WORDS(b-1, d)]
 *   signs    dev out, [N][TQ_SIGN_WORDS(d)]
 *   norms    dev out, [N] float32 ||x||
 *   rnorms   dev out, [N] float32 ||r||
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_quant_prod(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                  uint32_t* codes, uint32_t* signs, float* norms, float* rnorms, int64_t out_stride,
                  void* stream);

/*
 * tq_quant_prod_ws -- tq_quant_prod with a caller workspace (same outputs,
 * same passages).  For dimensions above 256 the tensor-core path computes the
 * QJL projection from the stored residual u = y - c[idx] (two fp16 pieces per
 * coordinate, 4 d_pad bytes per vector, d_pad = d rounded up to 128) so that
 * its fp32 sums stay of size ||u|| rather than ||x||; the workspace holds those
 * rows for up to ws_bytes / (4 d_pad) vectors (whole multiples of 128) at a
 * time and the call walks the batch in such chunks.  tq_quant_prod without a
 * workspace runs those dimensions on the CUDA cores instead.
 *   workspace, ws_bytes   dev scratch; tq_quant_prod_workspace(h, N) bytes run
 *            the batch in the fewest launches; any size of at least 512 d_pad
 *            bytes (128 vectors) is accepted; ignored (may be NULL) for d <= 256
 * Errors: as tq_quant_prod, plus TQ_EWORKSPACE (a non-NULL workspace below the
 * minimum).
 */
TQ_API int tq_quant_prod_ws(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                     uint32_t* codes, uint32_t* signs, float* norms, float* rnorms, int64_t out_stride,
                     void* workspace, size_t ws_bytes, void* stream);
/* Suggested workspace bytes for tq_quant_prod_ws (0 when none is used). */
TQ_API size_t tq_quant_prod_workspace(tq_handle h, int64_t N);

/*
 * tq_ip_scores -- estimated inner products of nq queries with N quantized vectors
 * ([tmdm, "双剑合璧", ✦ QJL]: the unbiased estimator corrects the quantization error
 * while the score is computed; [admirer, "內存價格能下來嗎？": nearest-neighbour search).
 *   TQ_PROD: s = n <Pi q, c[idx]> + rn sqrt(pi/2)/d <S q, sigma>, sigma_j = +-1
 *   TQ_MSE:  s = n <Pi q, c[idx]>
 * Each query is rotated (and projected) once.
 *   q        dev in, [nq][d] float32
 *   codes, signs, norms, rnorms   dev in, as written by tq_quant_* (signs and
 *            rnorms are ignored for TQ_MSE and may be NULL)
 *   scores   dev out, [nq][N] float32, or NULL when topk > 0 and only the
 *            top-k is wanted
 *   topk     0, or 1..TQ_MAX_TOPK: also write the topk largest scores per query
 *            to top_idx [nq][topk] int32 and top_val [nq][topk] float32, by
 *            score descending (ties: lower index first)
 *   workspace, ws_bytes   dev scratch of at least tq_ip_scores_workspace(...) bytes
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_EWORKSPACE, TQ_ECUDA.
 */
#define TQ_MAX_TOPK 64
TQ_API int tq_ip_scores(tq_handle h, const float* q, int64_t nq, const uint32_t* codes,
                 const uint32_t* signs, const float* norms, const float* rnorms, int64_t N,
                 float* scores, int topk, int32_t* top_idx, float* top_val, void* workspace,
                 size_t ws_bytes, void* stream);
TQ_API size_t tq_ip_scores_workspace(tq_handle h, int64_t nq, int64_t N, int topk);

/*
 * tq_attn_decode -- one decode step of attention over a TurboQuant K/V cache
 * ([tq.net, "实现步骤草图", 集成到 attention]: K and V are stored in TurboQuant form and
 * QJL is used inside attention; [tmdm, "实测数据"]: attention logits over a 4-bit cache).
 * For batch b, query head j (kv-head h = j / (Hq/Hkv)):
 *   logit_t = scale * est(q_bj, k_t)        (TQ_PROD estimator with handle hk)
 *   out_bj  = sum_t softmax(logit)_t * n_t Pi_V^T c_V[idx_t]   (values with hv, TQ_MSE)
 * The value sum runs in the rotated frame and Pi_V^T is applied once per output.
 *   hk, hv      TQ_PROD key handle and TQ_MSE value handle, same d
 *   q           dev in, [B][Hq][d] of q_dtype (TQ_F32 or TQ_BF16)
 *   B, Hq, Hkv  batch, query heads, kv-heads (Hq % Hkv == 0)
 *   T           context length (>= 1)
 *   kv_stride   token slots per (batch, kv-head) in the cache arrays (>= T):
 *               token t of (b, h) is row (b*Hkv + h)*kv_stride + t of
 *   kcodes [..][TQ_CODE_WORDS(bk-1, d)], ksigns [..][TQ_SIGN_WORDS(d)],
 *   knorms [..], krnorms [..], vcodes [..][TQ_CODE_WORDS(bv, d)], vnorms [..]
 *   scale       logit scale; Reading: the pages give none, callers pass 1/sqrt(d)
 *   out         dev out, [B][Hq][d] float32
 *   workspace   dev scratch of at least tq_attn_decode_workspace(...) bytes
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_EWORKSPACE, TQ_ECUDA.
 */
TQ_API int tq_attn_decode(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                   int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                   const float* knorms, const float* krnorms, const uint32_t* vcodes,
                   const float* vnorms, float scale, float* out, void* workspace, size_t ws_bytes,
                   void* stream);
TQ_API size_t tq_attn_decode_workspace(tq_handle hk, int B, int Hq, int Hkv, int64_t T);

/*
 * tq_attn_decode_static -- tq_attn_decode for callers that cannot allocate
 * device memory.  The paper has no counterpart to this call; it exists for
 * library users only.
 * Some callers may not allocate device memory while they run: a plugin whose
 * host application owns the whole device memory budget through its own pool
 * and gives the plugin no way to draw from it, or a service that must keep its
 * device footprint fixed once it has started.  They cannot provide the
 * workspace tq_attn_decode needs.  This call computes the same result with its
 * scratch in a fixed array compiled into the library instead, and allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *   Arguments and layouts: as tq_attn_decode, without workspace/ws_bytes.
 *   Limit: a shape whose tq_attn_decode_workspace(...) exceeds
 *   TQ_DECODE_STATIC_SCRATCH bytes is rejected with TQ_EWORKSPACE.
 *   The array (TQ_DECODE_STATIC_SCRATCH bytes) is held on every GPU that loads
 *   the library until the process exits.  The first call on a device looks up
 *   the array's device address (cudaGetSymbolAddress) with that device
 *   current; make that first call before any stream capture.  The address is
 *   kept for the life of the process: after a cudaDeviceReset both it and
 *   every handle of that device are stale and must not be used again.
 *   All calls on a device share the one array and it keeps the last call's
 *   contents; nothing in it has to start at zero (every scratch value is
 *   written before it is read within a call).  Calls that overlap on the GPU
 *   (different streams, or concurrent host threads) race on the array and
 *   must be serialised by the caller.
 * Errors: as tq_attn_decode, TQ_EWORKSPACE for shapes beyond the limit.
 */
#define TQ_DECODE_STATIC_SCRATCH (4 * 1024 * 1024)
TQ_API int tq_attn_decode_static(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int Hq,
                                 int Hkv, int64_t T, int64_t kv_stride, const uint32_t* kcodes,
                                 const uint32_t* ksigns, const float* knorms, const float* krnorms,
                                 const uint32_t* vcodes, const float* vnorms, float scale, float* out,
                                 void* stream);

/*
 * tq_attn_prefill -- attention of a block of nq new tokens (a prompt chunk)
 * over a TurboQuant K/V cache that already holds them ([tq.net, "实现步骤草图",
 * 集成到 attention]; [tmdm, "实测数据"]: logits over a 4-bit cache).  Token i of
 * the block sits at position T - nq + i and attends keys t <= T - nq + i
 * (causal); for batch b, token i, query head j (kv-head h = j / (Hq/Hkv)):
 *   out[b][i][j] = sum_{t <= T-nq+i} softmax(scale * est(q_bij, k_t)) n_t Pi_V^T c_V[idx_t]
 * The products run on the tensor cores (decoded keys and values as fp16
 * operands, fp32 accumulation); the value sum stays in the rotated frame and
 * Pi_V^T is applied once per output row.
 *   q         dev in, [B][nq][Hq][d] of q_dtype (TQ_F32 or TQ_BF16)
 *   T         context length including the block (nq <= T)
 *   kv_stride, cache arrays   as tq_attn_decode
 *   out       dev out, [B][nq][Hq][d] float32
 *   workspace dev scratch of at least tq_attn_prefill_workspace(...) bytes
 * Supported: d = 128, keys TQ_PROD b = 4, values TQ_MSE b = 4, Hq / Hkv a
 * divisor of 128, kv_stride % 4 == 0 (TQ_EUNSUPPORTED otherwise).
 * Range: the decoded operands are fp16 products n_k c[idx], rn_k and
 * n_v c_V[idx], so key norms, residual norms and value norms must stay below
 * 65504 / max|c| (about 3e5 for these codebooks); the kernel does not check it.
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_EWORKSPACE, TQ_ECUDA.
 */
TQ_API int tq_attn_prefill(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int nq, int Hq, int Hkv,
                           int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                           const float* knorms, const float* krnorms, const uint32_t* vcodes, const float* vnorms,
                           float scale, float* out, void* workspace, size_t ws_bytes, void* stream);
TQ_API size_t tq_attn_prefill_workspace(tq_handle hk, int B, int nq, int Hq, int Hkv, int64_t T);

/* ---------------------------------------------------------------- a cache split across devices */

/*
 * tq_attn_decode_partial -- the decode step of tq_attn_decode over the slice of
 * the context held here, stopped before normalisation so that slices held by
 * other devices can be combined with it ([tq.net, "实现步骤草图", 集成到 attention];
 * the split itself is not on the pages: one device's HBM is the limit of a
 * single cache).  For every (batch b, query head j) it writes the record
 *   partial[b*Hq + j] = (acc[0..d-1], m, l),  m = max_t logit_t (natural units),
 *   l = sum_t e^(logit_t - m),  acc = sum_t e^(logit_t - m) n_t c_V[idx_t]
 * with acc in the rotated value frame (Pi_V is not applied).  T = 0 (an empty
 * slice) writes acc = 0, m = -FLT_MAX, l = 0.
 *   arguments   as tq_attn_decode (T >= 0), with
 *   partial     dev out, [B*Hq][d + 2] float32
 *   workspace   dev scratch of at least tq_attn_decode_partial_workspace(...) bytes
 * Errors: as tq_attn_decode.
 */
TQ_API int tq_attn_decode_partial(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                                  int64_t T, int64_t kv_stride, const uint32_t* kcodes, const uint32_t* ksigns,
                                  const float* knorms, const float* krnorms, const uint32_t* vcodes,
                                  const float* vnorms, float scale, float* partial, void* workspace, size_t ws_bytes,
                                  void* stream);
TQ_API size_t tq_attn_decode_partial_workspace(tq_handle hk, int B, int Hq, int Hkv, int64_t T);

/*
 * tq_attn_merge -- combine the records of R slices and rotate back once:
 *   M = max_r m_r,  out = Pi_V^T (sum_r e^(m_r - M) acc_r) / (sum_r e^(m_r - M) l_r)
 *   hv        the TQ_MSE value handle of the records
 *   partials  dev in, [R][rows][d + 2] float32 (tq_attn_decode_partial's records
 *             of R slices, e.g. the result of an all-gather across devices)
 *   rows      B*Hq
 *   out       dev out, [rows][d] float32
 * A row whose slices are all empty has no softmax: its output is NaN.
 * Errors: TQ_EINVAL, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_attn_merge(tq_handle hv, const float* partials, int R, int64_t rows, float* out, void* stream);

/*
 * tq_topk_merge -- the global top-k of nq queries from R slices' own top-k
 * lists (the search of [admirer, "內存價格能下來嗎？"] over a database split across
 * devices, each scoring its slice with tq_ip_scores).
 *   val, idx    dev in, [R][nq][k] float32 scores and int32 indices local to each
 *               slice; a local index of INT32_MAX marks an empty candidate
 *   offsets     host in, [R]: the global index of each slice's first key
 *   out_idx, out_val   dev out, [nq][k]: by score descending, ties to the lower
 *               global index (INT32_MAX / -FLT_MAX where fewer than k candidates exist)
 * Errors: TQ_EINVAL (R outside 1..TQ_MAX_SHARDS, k outside 1..TQ_MAX_TOPK), TQ_EALIGN, TQ_ECUDA.
 */
#define TQ_MAX_SHARDS 64
TQ_API int tq_topk_merge(const float* val, const int32_t* idx, int R, int64_t nq, int k, const int64_t* offsets,
                         int32_t* out_idx, float* out_val, void* stream);

/* ---------------------------------------------------------------- a paged cache */

/*
 * tq_quant_paged -- quantize-on-write: quantize N vectors (tq_quant_mse /
 * tq_quant_prod with the handle's variant) and write vector i's outputs into
 * row slots[i] of the cache arrays, so a serving layer whose KV cache lives in
 * pages (a block table per sequence) stores each arriving token straight into
 * its page ([ttakun, "新旧量化方案深度权衡矩阵"]: each token is compressed as it
 * arrives; [tmdm, "实测数据"]: only the KV store and load change).
 *   x, dtype, N, x_stride   as tq_quant_mse (x_stride % 8 == 0 unless channels)
 *   channels   dev in, [d] int32, or NULL: vector i is x_i[channels[0..d-1]]
 *              (one channel group of a split cache, as tq_quant_gather)
 *   slots      dev in, [N] int64: the cache row of each vector (rows need not be
 *              distinct from earlier calls; two vectors of one call must not
 *              share a row)
 *   codes, signs, norms    dev out, cache arrays indexed by row as in tq_quant_prod
 *   rnorms     dev out, [rows] of rn_dtype: TQ_F32, or TQ_F16 -- the residual
 *              norm as one FP16 scalar per vector ([tq.net, "工程风险与应对",
 *              残差范数存储]), the nearest fp16 of the float32 result
 *   signs, rnorms are ignored for TQ_MSE handles (may be NULL)
 * Supported for d <= 256 (TQ_EUNSUPPORTED otherwise).
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN (x and slots 16-byte aligned,
 * the outputs 4-byte aligned), TQ_ECUDA.
 */
TQ_API int tq_quant_paged(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride, const int32_t* channels,
                          const int64_t* slots, uint32_t* codes, uint32_t* signs, float* norms, void* rnorms,
                          int rn_dtype, void* stream);

/*
 * tq_attn_decode_paged -- tq_attn_decode over a paged cache: token t of
 * (batch b, kv-head h) is row block_table[(b*Hkv + h)*max_pages + t / page_size]
 * * page_size + t % page_size of every cache array.
 *   block_table   dev in, [B*Hkv][max_pages] int32 page ids (max_pages *
 *                 page_size >= T)
 *   page_size     tokens per page, a multiple of 8
 *   krnorms       dev in, residual norms of rn_dtype (TQ_F32 or TQ_F16)
 *   other arguments as tq_attn_decode (every sequence has context length T)
 *   workspace     dev scratch of at least tq_attn_decode_workspace(hk, B, Hq, Hkv, T) bytes
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_EWORKSPACE, TQ_ECUDA.
 */
TQ_API int tq_attn_decode_paged(tq_handle hk, tq_handle hv, const void* q, int q_dtype, int B, int Hq, int Hkv,
                                int64_t T, const int32_t* block_table, int max_pages, int page_size,
                                const uint32_t* kcodes, const uint32_t* ksigns, const float* knorms,
                                const void* krnorms, int rn_dtype, const uint32_t* vcodes, const float* vnorms,
                                float scale, float* out, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- channel groups */

/*
 * tq_quant_gather -- quantize rows restricted to a list of channels:
 * vector i is (x_i[channels[0]], ..., x_i[channels[d-1]]), then exactly
 * tq_quant_mse / tq_quant_prod with the handle's variant.  Used to append a
 * token to a key cache whose channels are split into groups that are quantized
 * as separate instances (outlier channels at more bits, the rest at fewer:
 * [tq.net, "TurboQuant 最近的进展和外溢影响"]; 3.5 bits per channel and quantizing
 * each token as it arrives: [ttakun, "为什么TurboQuant把…"] / [ttakun, "新旧量化方案深度权衡矩阵"]).
 *   channels   dev in, [d] int32 channel indices into a row of x (x_stride wide)
 *   signs, rnorms  ignored (may be NULL) for TQ_MSE handles
 *   other arguments as tq_quant_prod, except that pointers need only be
 *   4-byte aligned (so codes/signs/norms may point at one token slot of a cache)
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_quant_gather(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride,
                           const int32_t* channels, uint32_t* codes, uint32_t* signs, float* norms, float* rnorms,
                           int64_t out_stride, void* stream);

/*
 * tq_quant_gather_groups -- tq_quant_gather for every channel group of a few
 * arriving tokens in one launch (the append of a split cache, [ttakun,
 * "新旧量化方案深度权衡矩阵"]: each token is compressed as it arrives).
 *   h          host array [ngroups] of handles (ngroups 1 or 2; d <= 256 each)
 *   channels   dev in, [sum d_g] int32: group g's channels at offset sum_{g'<g} d_g'
 *   codes, signs, norms, rnorms   host arrays [ngroups] of dev pointers, each
 *              as tq_quant_gather for that group (signs / rnorms entries may be
 *              NULL for TQ_MSE groups)
 *   N          vectors (0 <= N < 65536), x_stride, out_stride as tq_quant_gather
 * Pointers need only be 4-byte aligned.
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_quant_gather_groups(const tq_handle* h, int ngroups, const void* x, int dtype, int64_t N,
                                  int64_t x_stride, const int32_t* channels, uint32_t* const* codes,
                                  uint32_t* const* signs, float* const* norms, float* const* rnorms,
                                  int64_t out_stride, void* stream);

/*
 * tq_attn_logits -- attention logits over a TurboQuant_prod key cache whose
 * channels may be split into groups (the pages' outlier channels kept at
 * higher precision, [tq.net, "TurboQuant 最近的进展和外溢影响"]; logits over a
 * compressed cache, [tmdm, "实测数据"]).  For batch b, query head j
 * (kv-head h = j / 4, grouped-query attention with 4 query heads per kv-head):
 *   logits[b][j][t] = scale * sum_g est_g(q_bj[channels_g], k_{b,h,t,g})
 * with est_g the TurboQuant_prod estimator of group g's handle.
 *   hk         host array [ngroups] of TQ_PROD handles (1 group: d 64 or 128;
 *              2 groups: d = 64 each), mse bits 1..3
 *   channels   dev [sum d_g] int32: group g's channels of the query rows, at
 *              offset sum_{g'<g} d_g'; NULL allowed for one group with dq = d
 *   q          dev [B][Hq][dq] of q_dtype (TQ_F32 or TQ_BF16)
 *   Hq         must be 4 * Hkv
 *   kcodes, ksigns, knorms, krnorms   host arrays [ngroups] of dev pointers,
 *              each group's cache laid out as in tq_attn_decode (row
 *              (b*Hkv + h)*kv_stride + t)
 *   logits     dev out, [B][Hq][T] float32
 *   workspace  dev scratch of at least tq_attn_logits_workspace(...) bytes
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_EWORKSPACE, TQ_ECUDA.
 */
TQ_API int tq_attn_logits(const tq_handle* hk, int ngroups, const int32_t* channels, const void* q, int q_dtype,
                          int dq, int B, int Hq, int Hkv, int64_t T, int64_t kv_stride,
                          const uint32_t* const* kcodes, const uint32_t* const* ksigns,
                          const float* const* knorms, const float* const* krnorms, float scale, float* logits,
                          void* workspace, size_t ws_bytes, void* stream);
TQ_API size_t tq_attn_logits_workspace(const tq_handle* hk, int ngroups, int B, int Hq);

/* ---------------------------------------------------------------- PolarQuant */

/*
 * PolarQuant, the polar stage-one variant ([tmdm, "双剑合璧：PolarQuant + QJL",
 * ✦ PolarQuant]: after the random rotation the Cartesian coordinates become a
 * radius and a chain of bounded angles, so no normalisation constants are
 * stored; [admirer, "第一階段"]: coordinates are paired and mapped to polar
 * form, the pair radii are transformed the same way, recursively, down to one
 * final radius and a set of angles, each quantized with its own scalar
 * quantizer).  Readings (the pages give no grid or bit allocation): d a power
 * of two, L = log2 d levels; level-1 angles atan2(y_2i+1, y_2i) in [0, 2 pi)
 * take b1 bits on the uniform grid (cells [k, k+1) 2 pi / 2^b1, centroid in
 * the middle); an angle of level l >= 2, atan2(r_2i+1, r_2i) in [0, pi/2] of
 * the level below's radii, takes bh bits of the Lloyd-Max quantizer of its law
 * f_l ~ (sin t cos t)^(m-1), m = 2^(l-1) (sin^2 t ~ Beta(m/2, m/2) for a
 * uniform point on the sphere); the final radius is ||x|| (float32).  Values
 * on a threshold take the upper cell.  b1 = 4, bh = 2 spends about 3 bits per
 * coordinate.
 * Packed words per vector: TQ_POLAR_WORDS(b1, bh, d) = the d/2 level-1 codes in
 * the b1-bit layout of the code words above (as if they were d/2
 * coordinates), then the d/2 - 1 codes of levels 2..L (level 2 first, each
 * level in order) in the bh-bit layout.
 */
#define TQ_POLAR 2
#define TQ_POLAR_WORDS(b1, bh, d) (TQ_CODE_WORDS(b1, (d) / 2) + TQ_CODE_WORDS(bh, (d) / 2 - 1))

/*
 * tq_polar_codebook -- the scalar quantizer of one level's angles (host).
 *   b           bits, 1..8;  level  1..12
 *   centroids   host out [2^b] ascending; thresholds host out [2^b - 1] (may be NULL)
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED.
 */
TQ_API int tq_polar_codebook(int b, int level, double* centroids, double* thresholds);

/*
 * tq_create_polar -- a PolarQuant instance (variant TQ_POLAR).
 *   d    64 or 128;  b1   2 or 4 (level-1 bits);  bh   1 or 2 (bits of levels >= 2)
 *   Pi   host in [d*d] row-major float64 rotation (y = Pi x)
 * Allocates the handle's constants on the current device.
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_ENOMEM, TQ_ECUDA.
 */
TQ_API int tq_create_polar(tq_handle* h, int d, int b1, int bh, const double* Pi);

/*
 * tq_quant_polar -- PolarQuant codes of N vectors: n = ||x||, y = Pi x on the
 * tensor cores, the angle tree of y and each angle's cell (decided from the
 * squared radii and tangents, no trigonometry).
 *   x, dtype, N, x_stride, out_stride   as tq_quant_mse
 *   codes   dev out, row i at codes + i*out_stride*TQ_POLAR_WORDS(b1, bh, d)
 *   norms   dev out, float32, norms[i*out_stride]
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_quant_polar(tq_handle h, const void* x, int dtype, int64_t N, int64_t x_stride, uint32_t* codes,
                          float* norms, int64_t out_stride, void* stream);

/*
 * tq_dequant_polar -- x_hat = n Pi^T y_hat, y_hat the unit tree rebuilt from
 * the centroid angles (cos / sin products down the levels), on the tensor cores.
 *   codes [N][TQ_POLAR_WORDS(b1, bh, d)], norms [N]; out [N][d] of out_dtype
 * Errors: TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA.
 */
TQ_API int tq_dequant_polar(tq_handle h, const uint32_t* codes, const float* norms, int64_t N, void* out,
                            int out_dtype, void* stream);

/* ---------------------------------------------------------------- diagnostics */

/*
 * tq_device_status -- read and clear the handle's device status word
 * (synchronous: waits for the device).  0 = no event.  A kernel that sets a
 * bit has left before writing all of its outputs, and the call that launched
 * it has returned TQ_OK: callers that need to know poll this word.  Bit 0 (TQ_STATUS_TIMEOUT): a tensor-core
 * kernel gave up a wait on one of its own pipeline barriers after ~2 s and
 * returned early; its outputs for that call are incomplete.  Bit 1
 * (TQ_STATUS_LAYOUT): a decode or logits kernel built for the shared-memory
 * address that tq_create measured found its dynamic shared window elsewhere
 * and returned without writing its outputs.
 * Errors: TQ_EINVAL, TQ_ECUDA.
 */
#define TQ_STATUS_TIMEOUT 1
#define TQ_STATUS_LAYOUT 2
TQ_API int tq_device_status(tq_handle h, int* status);

/* tq_last_error -- message of the last failing call on this thread ("" if none). */
TQ_API const char* tq_last_error(void);

/* tq_version -- library version string. */
TQ_API const char* tq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
