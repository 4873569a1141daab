/*
 * slim.h - C ABI of libslim, a B200 (sm_100a) implementation of the per-layer
 * quantize path of SliM-LLM (salience-driven group-wise mixed-precision
 * post-training quantization of LLM weights).
 *
 * Sources that define the operations (web pages about the method):
 *   [P1] rkmt.cn, "【ICML 2025】SliM-LLM 论文解读", sections 核心设计
 *        (组件一 SBA, 组件二 SQC), 实验设计与结果 (评测协议), FAQ.
 *   [P2] atlas.scime.ai summary of the SliM-LLM paper, section Approach.
 *   [P3] briefgpt.xyz, arXiv 2405.14917 abstract.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - W is the layer weight, float32, m x n, row-major (out x in, the layout of
 *   a PyTorch Linear). X is the calibration activations, N x n, row-major,
 *   float32 (SLIM_X_F32) or bf16 bit patterns (SLIM_X_BF16).
 * - Columns are split into k = n / group consecutive groups; group is 32, 64
 *   or 128 and must divide n. avg_bits is the average bit-width b (2..7); the
 *   groups get b-1, b or b+1 bits.
 * - Every array argument is DEVICE memory owned by the caller unless marked
 *   HOST. The library keeps no data between calls and never frees caller
 *   memory; it caches, per host thread and device, a few CUDA streams and
 *   events and the inverse stage's CUDA graph (created on first use, kept
 *   until the process exits). Work on those side streams is ordered after
 *   `stream` and joined back into it before the call returns. Arrays must
 *   not overlap. W must be 16-byte aligned and X too.
 * - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   Work is ordered on it. Each call enqueues its kernels, then waits for the
 *   stream to drain and reads the call's device status word, so that it can
 *   return device-side failures (SLIM_ENOTPD, SLIM_ETIMEOUT). Outputs are
 *   complete when the call returns SLIM_OK.
 * - Workspace: `ws` is device scratch of at least the size the matching
 *   *_workspace_bytes function returns, 256-byte aligned. ws == NULL makes the
 *   call allocate it (cudaMallocFromPoolAsync on `stream`) and free it itself,
 *   from a memory pool the library creates per device on first use and keeps
 *   until the process exits (freed blocks stay in that pool for the next call).
 *   The device's default pool and its settings are not touched.
 * - Per-device state (the pool, cached streams, events and graphs, the address
 *   of slim_salience_noalloc's array) is created on first use on a device; a
 *   cudaDeviceReset of that device invalidates it, so a process that resets a
 *   device must not call the library on that device again.
 * - Errors are returned, never raised: on any status other than SLIM_OK the
 *   outputs are unspecified. Arguments are validated before any launch.
 * - Calls on the same device that share a workspace must not overlap.
 */
#ifndef SLIM_H
#define SLIM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SLIM_OK = 0,
  SLIM_EINVAL = 1,    /* bad argument (size, group, bits, NULL pointer, alignment) */
  SLIM_ENOMEM = 2,    /* the library could not allocate device memory */
  SLIM_ECUDA = 3,     /* a CUDA runtime call failed; see slim_last_cuda_error() */
  SLIM_ETIMEOUT = 4,  /* a device-side wait ran past its limit; the kernel stopped */
  SLIM_ENOTPD = 5,    /* the damped Hessian has no Cholesky factor */
  SLIM_ENODEV = 6,    /* no sm_100 device is current */
  SLIM_EINJECTED = 7, /* a failure was injected on the host (SLIM_FAULT=<stage>) */
  SLIM_ERANGE = 8     /* an input does not fit the fp16 tensor-core operands of the
                         SBA scoring (|x| or 256 |w| above 65504) */
} slim_status;

typedef enum { SLIM_X_F32 = 0, SLIM_X_BF16 = 1 } slim_xdtype;

/* How SBA scores a candidate allocation. SLIM_OBJ_KL is the method's
 * objective ([P1] 组件一 SBA: output KL divergence). SLIM_OBJ_MSE, the mean
 * squared error of the layer outputs, is the objective the method is compared
 * against in its ablation ([P2] Measured effects: KL rather than MSE). */
typedef enum { SLIM_OBJ_KL = 0, SLIM_OBJ_MSE = 1 } slim_objective;

/* Operand precision of the SBA scoring's weight side (bf16 X). Each 64-column
 * box of the weight-side arrays is an fp16 value (11 significant bits) or an
 * fp16 hi/lo pair (22 bits, twice the tensor-core work on that box).
 * SLIM_SBA_ADAPTIVE pairs the boxes that carry the most output rounding error:
 * per box the estimate sum_j |x_j|^2 |w_j|^2 (column energies of W and of the
 * first 16384 tokens of X) is ranked, and boxes are paired in descending order
 * until at most 1/32 of the total estimate is left; with activation-outlier
 * channels that is typically the few boxes holding them. SLIM_SBA_FULL pairs
 * every box. fp32 X always takes every box in three parts (X hi/lo x weight
 * hi/lo, less the lo x lo product). */
typedef enum { SLIM_SBA_ADAPTIVE = 0, SLIM_SBA_FULL = 1 } slim_sba_precision;

/* Human-readable text of a status code. Never NULL. */
const char* slim_status_string(int status);
/* Text of the last CUDA error seen by this thread's calls ("" if none). */
const char* slim_last_cuda_error(void);
/* The device-side detail of this host thread's last failed call's status:
 * for SLIM_ENOTPD the pivot index; for SLIM_ETIMEOUT the id of the bounded
 * wait that gave up (kernel-specific); for SLIM_ERANGE where the value was
 * found. 0 after a call that succeeded on the device. */
int slim_last_status_detail(void);
/* Library version string. */
const char* slim_version(void);

/* Measured fp64 rates of the current device in TFLOP/s: the fp64 tensor-core
 * MMA (m8n8k4) and the fp64 FMA pipe, each the best of three short runs of
 * independent chains on every SM (a few milliseconds in all). Not an operation
 * of the method: the roofline denominators of its fp64 stages (the inverse
 * Hessian, the GPTQ update, SQC). Waits for `stream`. */
int slim_peak_fp64(double* dmma_tflops, double* dfma_tflops, void* stream);

/* Number of SBA candidates, floor(k / 2) + 1 ([P1] 组件一 SBA: the search
 * range of the promoted-group count p is [0, k/2]). */
int slim_num_candidates(int64_t n, int group);

/* Packed-code words per row: n * avg_bits / 32. */
int64_t slim_row_words(int64_t n, int avg_bits);

/* Number of CUDA kernels this library has launched in this process so far
 * (all threads, all calls). Differences around a call count its launches. */
int64_t slim_launch_count(void);

/* ------------------------------------------------------------------------
 * slim_hessian: H = 2 X^T X ([P1] 组件一 SBA: the Hessian is approximated
 * from calibration activations, no backpropagation).
 *   X   device, N x n, row-major, dtype xdtype.
 *   H   device, n x n float64, row-major; both triangles are written.
 * bf16 X runs on the tensor cores (tcgen05, fp32 accumulation over token
 * slices, fp64 sum of the slices); float32 X runs an fp64-accumulating
 * CUDA-core kernel. Requires n % 32 == 0 and N >= 1.
 */
size_t slim_hessian_workspace_bytes(int64_t N, int64_t n, int xdtype);
int slim_hessian(const void* X, int xdtype, int64_t N, int64_t n, double* H,
                 void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * slim_hinv_diag: h_j = [H_d^-1]_jj, the inverse-Hessian diagonal used by the
 * salience formula ([P1] 组件一 SBA, delta formula).
 *   H_d = H with every zero diagonal entry set to 1, plus
 *         alpha * mean(diag) on the diagonal (alpha = 0.01 is the usual damping).
 *   H   device, n x n float64 row-major, read only (symmetric; the lower
 *       triangle is used).
 *   h   device, n float64.
 * Blocked fp64 Cholesky H_d = L L^T, blocked inverse of L, then column sums
 * of squares of L^-1. Returns SLIM_ENOTPD if a pivot is not positive.
 */
size_t slim_hinv_diag_workspace_bytes(int64_t n);
int slim_hinv_diag(const double* H, int64_t n, double alpha, double* h,
                   void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * slim_salience: delta_ij = w_ij^2 / h_j^2 ([P1] 组件一 SBA), group means
 * S_c = mean over rows and the group's columns ([P2] Approach: allocation by
 * average group salience), and the groups in descending S (equal values: the
 * lower group index first).
 *   W      device m x n float32;  h device n float64.
 *   S      device k float64;      order device k int32.
 */
size_t slim_salience_workspace_bytes(int64_t m, int64_t n, int group);
int slim_salience(const float* W, int64_t m, int64_t n, const double* h, int group,
                  double* S, int32_t* order, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * slim_salience_noalloc: the same computation and outputs as slim_salience,
 * for callers that cannot allocate device memory. The pages have no
 * counterpart; it is a deployment variant. Some callers may not call
 * cudaMalloc or let a library do so: code that runs inside an engine that owns
 * every byte of device memory through its own pool and budget, code on a path
 * where the implicit device synchronization of cudaMalloc/cudaFree is not
 * acceptable, or code under a fixed memory cap planned in advance. This entry
 * point allocates nothing: its scratch is a fixed 256 KiB device array inside
 * the library (held on every GPU that loads the library until the process
 * exits), enough for n <= 32768 input columns; larger n returns SLIM_EINVAL.
 * The first call on a device also looks up that array's device address. All
 * calls on a device
 * share the array: calls that overlap on the GPU race and must be serialized
 * by the caller. The call waits for `stream` to drain before returning.
 */
int slim_salience_noalloc(const float* W, int64_t m, int64_t n, const double* h, int group,
                          double* S, int32_t* order, void* stream);

/* ------------------------------------------------------------------------
 * slim_sba_search: salience-determined bit allocation ([P1] 组件一 SBA,
 * [P2] Approach). For p = 0 .. floor(k/2): groups order[0..p) get avg_bits+1,
 * groups order[k-p..k) get avg_bits-1, the rest avg_bits (balanced counts, so
 * the average stays avg_bits). Each candidate is scored by
 *   KL_p = mean over the N tokens of KL(softmax(x W^T) || softmax(x W_p^T)),
 * softmax over the m output features, W_p the per-group min-max round-to-
 * nearest dequantization of W under that allocation. p* is the smallest p
 * with the least KL.
 *   order    device k int32 (from slim_salience): a permutation of 0..k-1,
 *            checked on the device (otherwise SLIM_EINVAL).
 *   kl       device P float64 (P = slim_num_candidates), may be NULL.
 *   p_star   device int32, may be NULL.
 *   bits     device k uint8 (the allocation at p*).
 * All candidates are scored in one pass over X: a tensor-core kernel keeps,
 * per token tile, the outputs X W^T and the quantization-error outputs in
 * tensor memory, and updates them group pair by group pair as p grows. The
 * tensor-core operands are fp16: X converted from bf16 (exact for
 * |x| >= 2^-17; smaller values round to fp16 subnormals, an absolute error
 * below 2^-25) or split into two fp16 parts when fp32; each weight-side array
 * scaled by 2^8, as fp16 values, with the boxes that carry most of the
 * rounding error held as fp16 hi/lo pairs (22 significant bits; see
 * slim_sba_precision). Inputs with |x| > 65504 or |w| > 255 return
 * SLIM_ERANGE.
 */
size_t slim_sba_workspace_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group);
int slim_sba_search(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N,
                    int group, int avg_bits, const int32_t* order, double* kl, int32_t* p_star,
                    uint8_t* bits, void* ws, size_t ws_bytes, void* stream);

/* slim_sba_search with the scoring objective and the operand precision
 * selectable: objective is a slim_objective, precision a slim_sba_precision
 * (slim_sba_search uses SLIM_OBJ_KL, SLIM_SBA_ADAPTIVE). With SLIM_OBJ_MSE, kl receives per candidate the mean over
 * tokens and outputs of (x W_p^T - x W^T)^2 and p* minimises it. The order
 * argument is any permutation of the groups: the salience order is the
 * method; 0, 1, ..., k-1 (promote the first groups, demote the last) is the
 * head-tail allocation and a random permutation the random allocation of the
 * method's ablation ([P1] Fig. 5 caption: random / head-tail allocation;
 * [P2] Measured effects). Workspace: slim_sba_workspace_bytes. */
int slim_sba_search_ex(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N,
                       int group, int avg_bits, const int32_t* order, int objective, int precision,
                       double* kl, int32_t* p_star, uint8_t* bits, void* ws, size_t ws_bytes,
                       void* stream);

/* ------------------------------------------------------------------------
 * slim_sba_search_split: slim_sba_search's outputs, bit for bit, from a
 * schedule in two parts. The first part (per token tile: the outputs x W^T
 * and the error outputs of the base allocation, over the whole input width)
 * does not use the salience order; it runs token chunk by token chunk
 * (chunk_tokens, a positive multiple of 256, each chunk launched on its own)
 * and keeps each tile's state in the workspace (8 bytes per token and
 * output). The candidate steps then continue from that state. This is the
 * schedule slim_quantize_layer_host runs under its host-to-device copy of X
 * (the first part of each chunk as soon as the chunk lands); here it is
 * callable on its own. Arguments and errors as slim_sba_search; ws NULL
 * allocates. Workspace: slim_sba_split_workspace_bytes.
 */
size_t slim_sba_split_workspace_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group);
int slim_sba_search_split(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N,
                          int group, int avg_bits, const int32_t* order, double* kl, int32_t* p_star,
                          uint8_t* bits, int64_t chunk_tokens, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * slim_sqc: salience-weighted quantizer calibration ([P1] 组件二 SQC,
 * [P2] Approach, [P3]). For each (row i, group c) with b = bits[c]:
 *   mask   w < mu - 3 sigma or w > mu + 3 sigma (population sigma);
 *   s0, z0 min-max scale (hi - lo)/(2^b - 1) and float zero -lo/s0;
 *   tau_t  = (1 - lambda) + 2 lambda t / (n_tau - 1), t < n_tau (tau = 1 if n_tau = 1);
 *   q      = clamp(rint(w / (tau_t s0) + z0), 0, 2^b - 1), w_hat = tau_t s0 (q - z0);
 *   E_t    = mean_{mask} delta e^2 + mean_{not mask} delta e^2, e = w - w_hat,
 *            delta = w^2 / h_j^2;
 *   t*     = the smallest t with the least E_t (all arithmetic in fp64).
 * Outputs:
 *   codes    device uint32, m x slim_row_words(n, avg_bits): row i is a
 *            little-endian bit stream; group c's g codes (bits[c] bits each,
 *            column order, least significant bit first) follow the groups
 *            before it. sum(bits) must equal k * avg_bits.
 *   scale, zero  device m x k float32 (w_hat = scale * (q - zero)).
 *   tau_idx  device m x k uint8 (t*), may be NULL.
 * A group whose values are all equal stores scale 1, zero -lo, codes 0, t* 0.
 * Requires n_tau in [1, 256], 0 <= lambda < 1. lambda is taken as given
 * (double), so the tau grid is the exact fp64 expression above.
 */
int slim_sqc(const float* W, int64_t m, int64_t n, const double* h, const uint8_t* bits,
             int group, int avg_bits, double lambda, int n_tau, uint32_t* codes, float* scale,
             float* zero, uint8_t* tau_idx, void* stream);

/* ------------------------------------------------------------------------
 * slim_gptq: the quantization of slim_sqc inside the GPTQ layer loop ([P1]
 * 核心设计: SliM-LLM inserts its two components into GPTQ's layer-wise
 * quantization skeleton; [P1] FAQ). Columns are taken in order. When the loop
 * reaches the first column of group c, the group's quantizer is calibrated as
 * slim_sqc does (bits[c], 3-sigma mask, tau search, element salience w^2/h_j^2
 * with h = diag(H_d^-1)) on the group's weights as the compensation of the
 * earlier columns has left them; each column is then rounded with its group's
 * quantizer, and its error divided by U_jj is subtracted, times row j of U,
 * from the later columns, where H_d^-1 = U^T U (U upper triangular, H_d = H
 * with zero diagonal entries set to 1 plus 0.01 mean(diag) on the diagonal).
 * All arithmetic is fp64; the later columns take each 128-column block's
 * errors at once (the same sums regrouped).
 *   H        device n x n float64 (slim_hessian), read only.
 *   bits     device k uint8 (slim_sba_search), summing to k * avg_bits.
 *   codes, scale, zero, tau_idx: as slim_sqc (tau_idx may be NULL).
 * Requires m <= 65535 * 64. Returns SLIM_ENOTPD if H_d has no Cholesky factor.
 * Workspace: slim_gptq_workspace_bytes (about 8 (2 n^2 + m n) bytes plus the
 * inverse stage's scratch); ws NULL allocates.
 */
size_t slim_gptq_workspace_bytes(int64_t m, int64_t n);
int slim_gptq(const float* W, int64_t m, int64_t n, const double* H, const uint8_t* bits, int group,
              int avg_bits, double lambda, int n_tau, uint32_t* codes, float* scale, float* zero,
              uint8_t* tau_idx, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * slim_dequant_gemv: y = x W_hat^T on the packed layer, the inference product
 * whose token rate on current GPU kernels the pages name as the method's
 * limitation for mixed 1/2/3-bit groups ([P1] 局限性; [P2] Limitations).
 * W_hat[i][j] = scale[i][c] (q_ij - zero[i][c]) with q_ij the code of column j
 * (group c = j / group) in the layout of slim_sqc.
 *   codes    device m x slim_row_words(n, avg_bits) uint32 (16-byte aligned).
 *   bits     device k uint8, each in 1..8, summing to k * avg_bits (the
 *            caller's precondition: the kernel reads no word outside a row
 *            whatever bits holds, but y is then unspecified).
 *   scale, zero  device m x k float32.
 *   x        device batch x n, row-major, float32 or bf16 (xdtype).
 *   y        device batch x m float32.
 * batch is 1..8. Arithmetic: fp32. Per row, group c of width b and token,
 * A = sum_j x_j (1 + q_j 2^-b) and xs = sum_j x_j, and y gains
 * scale (2^b (A - xs) - zero xs), which is sum_j x_j W_hat[i][j] regrouped;
 * the groups' terms are added in a fixed order, so repeated calls on the same
 * inputs return the same y. The call is asynchronous: it returns once the kernels are enqueued on `stream` (host-side
 * argument checks only), so decode loops can issue it back to back. Workspace:
 * slim_dequant_gemv_workspace_bytes (0 when one launch covers every group of a
 * row, as for the usual layer shapes); ws NULL takes it from the library's
 * pool and returns it in stream order.
 */
size_t slim_dequant_gemv_workspace_bytes(int64_t m, int64_t n, int group, int avg_bits, int64_t batch);
int slim_dequant_gemv(const uint32_t* codes, const uint8_t* bits, const float* scale, const float* zero,
                      int64_t m, int64_t n, int group, int avg_bits, const void* x, int xdtype,
                      int64_t batch, float* y, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * slim_quantize_layer: the whole path, hessian -> hinv_diag -> salience ->
 * sba_search -> sqc ([P1] 核心设计: SBA allocates bits between groups, SQC
 * calibrates each group's quantizer), with damping alpha = 0.01.
 *   codes, scale, zero: as slim_sqc.  bits: device k uint8.
 */
size_t slim_workspace_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group, int avg_bits);
int slim_quantize_layer(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N,
                        int group, int avg_bits, double lambda, int n_tau, uint32_t* codes,
                        float* scale, float* zero, uint8_t* bits, void* ws, size_t ws_bytes,
                        void* stream);

/* Optional diagnostics of slim_quantize_layer_ex. Pointers may be NULL. */
typedef struct {
  double* H;          /* device n x n float64 */
  double* h;          /* device n float64 */
  double* S;          /* device k float64 */
  int32_t* order;     /* device k int32 */
  double* kl;         /* device P float64 */
  uint8_t* tau_idx;   /* device m x k uint8 */
  int32_t p_star;     /* HOST, written by the call */
  float stage_ms[8];  /* HOST, written: stages hessian, hinv_diag, salience, sba_search, sqc,
                         total, then the tensor-core kernels alone: hessian (bf16 X), sba scoring */
  uint8_t* sba_split; /* device (n + 63) / 64 uint8: 1 for the 64-column boxes the SBA scoring
                         took as fp16 hi/lo pairs (see slim_sba_precision) */
} slim_diag;

int slim_quantize_layer_ex(const float* W, int64_t m, int64_t n, const void* X, int xdtype,
                           int64_t N, int group, int avg_bits, double lambda, int n_tau,
                           uint32_t* codes, float* scale, float* zero, uint8_t* bits, void* ws,
                           size_t ws_bytes, void* stream, slim_diag* diag);

/* Variants of the whole path, for the method's ablations. A zeroed struct (or
 * opt == NULL) is the method itself. */
typedef struct {
  int objective;         /* slim_objective of the SBA search (default SLIM_OBJ_KL) */
  int sba_precision;     /* slim_sba_precision of the SBA search (default SLIM_SBA_ADAPTIVE) */
  int gptq;              /* 0: SQC on the weights as they are (default); 1: the GPTQ column loop
                            with error compensation (slim_gptq) in place of that SQC stage */
  const int32_t* order;  /* device k int32, or NULL for the salience order. A caller's
                            permutation of the groups replaces the salience order in the
                            search (see slim_sba_search_ex: head-tail, random). Checked on
                            the device (SLIM_EINVAL if not a permutation). Must not be
                            diag->order. diag->order then returns this order. */
} slim_options;

/* slim_quantize_layer_ex with options (opt may be NULL). Workspace:
 * slim_workspace_bytes. */
int slim_quantize_layer_opts(const float* W, int64_t m, int64_t n, const void* X, int xdtype,
                             int64_t N, int group, int avg_bits, double lambda, int n_tau,
                             uint32_t* codes, float* scale, float* zero, uint8_t* bits, void* ws,
                             size_t ws_bytes, void* stream, const slim_options* opt, slim_diag* diag);

/* ------------------------------------------------------------------------
 * slim_quantize_layer_host: slim_quantize_layer on HOST arrays (W, X in;
 * codes, scale, zero, bits out; same layouts). The call allocates device
 * buffers, copies inputs to the device, runs the path, copies results back
 * and frees. Pinned host memory makes the copies asynchronous-capable and
 * fast; pageable memory works too.
 */
int slim_quantize_layer_host(const float* W, int64_t m, int64_t n, const void* X, int xdtype,
                             int64_t N, int group, int avg_bits, double lambda, int n_tau,
                             uint32_t* codes, float* scale, float* zero, uint8_t* bits,
                             void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SLIM_H */
