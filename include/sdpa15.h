/*
 * sdpa15.h -- C ABI of a B200 (sm_100a) scaled dot-product attention forward.
 *
 * The operation (exactref.ai, "scaled_dot_product_attention", sections
 * "Arguments" and "Full specification"):
 *
 *     O   = softmax(Q K^T * scale + mask) V        over the key axis
 *     lse = log(sum_j exp(logit_ij))               natural log, per query row
 *
 * - scale: when has_scale == 0 it is 1/sqrt(E), applied exactly once to the
 *   raw dot products; an explicit scale (e.g. 1/E, or 1.0 for a query that was
 *   pre-scaled by the caller) is used as given.  Pre-scaling Q and also taking
 *   the default gives the double-scaled 1/E attention of the hourtab.com
 *   xFormers post ("Why double scaling makes attention uniform").
 * - mask kinds: NONE; CAUSAL keeps key j for query i iff j <= i (top-left
 *   aligned when L != S); BLOCK_DIAG / BLOCK_DIAG_CAUSAL restrict every query
 *   of a packed batch to the keys of its own segment (xFormers
 *   BlockDiagonalMask / BlockDiagonalCausalMask, insureai360 tutorial section
 *   4 "Variable-length packed batch"); FLOAT_BIAS adds a float32 bias to the
 *   scaled scores, -inf removing a key; BOOL reads one byte per (b, h, i, j),
 *   nonzero where query i may see key j, and acts as a 0 / -inf bias (so a
 *   NaN score under a removed key still makes its row NaN, as a bias would).
 * - GQA (exactref "Arguments", enable_gqa; the BMGHK layout of the tutorial's
 *   section 5): Hq is a multiple of Hkv and query head h reads key/value head
 *   h / (Hq / Hkv).
 * - lse is float32 for every input dtype: exactref "logsumexp and its
 *   format" computes it in float32 for the 16-bit formats and in the input's
 *   own format otherwise, which here is float32 too.  A row that sees no key gets O = 0 and lse = -inf; a NaN input
 *   turns its row into NaN (exactref "Special values and dropout").
 *
 * Memory and threading contract of every entry point below:
 * - All tensor pointers are DEVICE pointers on the current CUDA device.  The
 *   caller owns and allocates every buffer, the workspace included; the
 *   library allocates no device memory on this path and never synchronises:
 *   work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *   stream) and the call returns once it is enqueued.
 * - Strides are in ELEMENTS, four per tensor, in the order
 *   (batch, head, sequence, feature).  BHLE (B,H,L,E) and BMHK (B,M,H,K)
 *   layouts are both expressed this way.  The feature stride must be 1.
 * - Errors are returned as sdpa_status codes; nothing traps or aborts.  On an
 *   error no work has been enqueued, except SDPA_ERR_CUDA, which reports a
 *   failed launch.
 */
#ifndef SDPA15_H
#define SDPA15_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SDPA_OK = 0,
  SDPA_ERR_INVALID = 1,     /* bad argument: null pointer, shape, stride, GQA ratio, cu_seqlens, dtype */
  SDPA_ERR_UNSUPPORTED = 2, /* well-formed but not implemented: E outside 0..256 or Ev outside 1..256, not an sm_100 device */
  SDPA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  SDPA_ERR_WORKSPACE = 4    /* workspace missing or smaller than sdpa_fwd_workspace_size() */
} sdpa_status;

typedef enum { SDPA_F32 = 0, SDPA_F16 = 1, SDPA_BF16 = 2 } sdpa_dtype;

typedef enum {
  SDPA_MASK_NONE = 0,
  SDPA_MASK_CAUSAL = 1,
  SDPA_MASK_BLOCK_DIAG = 2,
  SDPA_MASK_BLOCK_DIAG_CAUSAL = 3,
  SDPA_MASK_FLOAT_BIAS = 4,
  SDPA_MASK_BOOL = 5
} sdpa_mask_kind;

/* Version of this ABI (changes when a signature or an enum changes). */
int sdpa_abi_version(void);

/* Human-readable name of a status code (a static string; never NULL). */
const char* sdpa_status_string(int status);

/*
 * Bytes of device workspace sdpa_fwd() needs for this problem (0 when it needs
 * none).  Depends only on the arguments; the same arguments always give the
 * same size.  Pass a workspace of at least this many bytes, 256-byte aligned.
 * Returns 0 for arguments sdpa_fwd() would reject.
 */
size_t sdpa_fwd_workspace_size(int B, int Hq, int Hkv, int L, int S, int E, int Ev,
                               int mask_kind, int dtype);

/*
 * Attention forward: out = softmax(q k^T * scale + mask) v, lse = per-row
 * logsumexp of the logits.
 *
 * q     [B, Hq,  L, E ]  dtype, strides q_stride   (elements)
 * k     [B, Hkv, S, E ]  dtype, strides k_stride
 * v     [B, Hkv, S, Ev]  dtype, strides v_stride
 * out   [B, Hq,  L, Ev]  dtype, strides o_stride   (written)
 * lse   [B, Hq,  L]      float32, contiguous       (written)
 * dtype             SDPA_F32, SDPA_F16 or SDPA_BF16 (q, k, v and out share it)
 * has_scale, scale  has_scale == 0: scale = 1/sqrt(E); else `scale` as given
 *                   (any finite value, 0 included)
 * E = 0             allowed: the scores are empty sums, so the logits are
 *                   the mask alone (exactref "Full specification"); q and k
 *                   may then be NULL.
 * mask_kind         sdpa_mask_kind
 * cu_seqlens        BLOCK_DIAG*: device int32[n_seqs + 1], cumulative segment
 *                   starts of one packed batch: cu[0] = 0, non-decreasing,
 *                   cu[n_seqs] = L = S, and B must be 1.  Otherwise ignored.
 *                   The kernels clamp every segment to [0, L), so a malformed
 *                   array cannot make them read or write out of bounds.
 * n_seqs            number of segments (>= 1) for BLOCK_DIAG*
 * max_seqlen        BLOCK_DIAG*: an upper bound on the segment lengths (the
 *                   grid is sized from it; segments longer than it are an
 *                   error the kernels cannot detect and leave rows unwritten)
 * bias, bias_stride FLOAT_BIAS: device float32 [B, Hq, L, S] with element
 *                   strides (b, h, l, s); 0 broadcasts an axis.  BOOL: device
 *                   bytes (nonzero = the key is visible) of the same shape,
 *                   strides in bytes.  Else ignored.
 * workspace         device scratch of sdpa_fwd_workspace_size() bytes (may be
 *                   NULL when that size is 0); its contents need no clearing
 *                   and are garbage afterwards.
 * stream            cudaStream_t to enqueue on.
 *
 * Returns SDPA_OK or an error status (see sdpa_status).
 */
int sdpa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
             int B, int Hq, int Hkv, int L, int S, int E, int Ev,
             const int64_t q_stride[4], const int64_t k_stride[4],
             const int64_t v_stride[4], const int64_t o_stride[4],
             int has_scale, float scale,
             int mask_kind, const int32_t* cu_seqlens, int n_seqs, int max_seqlen,
             const void* bias, const int64_t bias_stride[4],
             int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Which kernel family sdpa_fwd() would run for these arguments (no work is
 * done): 1 = tcgen05/TMA prefill, 2 = split-S decode + combine, 3 = general
 * SIMT kernel, or a negative sdpa_status for rejected arguments.  For tests
 * and benchmarks that must know the path taken.
 */
int sdpa_fwd_plan(int B, int Hq, int Hkv, int L, int S, int E, int Ev,
                  const int64_t q_stride[4], const int64_t k_stride[4],
                  const int64_t v_stride[4], const int64_t o_stride[4],
                  int mask_kind, int dtype,
                  const void* q, const void* k, const void* v, const void* out);

/*
 * Number of kernels the last successful sdpa_fwd() or sdpa_decode_paged()
 * call on this host thread enqueued (1 or 2), for launch accounting in benchmarks.
 */
int sdpa_last_launch_count(void);

/*
 * Reads and clears the device-side error words of the current device
 * (synchronises the device).  *code receives 0 when no kernel reported an
 * error.  Codes below 30 mean a kernel's bounded wait on one of its own
 * pipeline barriers ran out (2 s) and its outputs for that launch are not
 * valid; 31 and 32 are sdpa_decode_paged()'s checks of seq_lens and of the
 * block table.  Returns SDPA_OK, SDPA_ERR_INVALID for a NULL `code`, or
 * SDPA_ERR_CUDA.
 */
int sdpa_take_device_error(int* code);

/*
 * Bytes of workspace sdpa_bwd() needs (0 for rejected shapes): one float32
 * per (batch, query head, query row), rounded up to 256 bytes.
 */
size_t sdpa_bwd_workspace_size(int B, int Hq, int Hkv, int L, int S, int E, int Ev,
                               int mask_kind, int dtype);

/*
 * Gradients of the attention forward (exactref.ai
 * "scaled_dot_product_attention", section "er.scaled_dot_product_attention.
 * backward"): for the output gradient `dout`, with P the forward's weights,
 *   dP = dout V^T,  D_i = sum_j P_ij dP_ij,  dS = P * (dP - D),
 *   dv = P^T dout,  dq = scale * dS K,  dk = scale * dS^T Q,
 * with dk and dv summed over the query heads that share a key/value head.
 *
 * q, k, v          the forward's inputs, as for sdpa_fwd().
 * out, lse         the forward's outputs for these inputs (out in the input
 *                  dtype with o_stride; lse float32 contiguous (B, Hq, L)).
 *                  P is recomputed as exp(logit - lse); D_i is computed as
 *                  dout_i . out_i, equal to sum_j P_ij dP_ij.
 * dout             output gradient, the shape and dtype of out, element
 *                  strides do_stride[4] (batch, head, seq, feature).
 * dq, dk, dv       gradients, written (not accumulated) in the input dtype,
 *                  shapes of q, k, v, element strides dq_stride, dk_stride,
 *                  dv_stride.  Every element is written exactly once.
 * B..Ev, strides of q/k/v/out, has_scale/scale, mask_kind, cu_seqlens,
 * n_seqs, max_seqlen, bias, bias_stride, dtype: as for sdpa_fwd(); the float
 * bias gets no gradient.
 * workspace        device memory of at least sdpa_bwd_workspace_size()
 *                  bytes, 256-byte aligned, owned by the caller.
 * stream           cudaStream_t to enqueue on; nothing synchronises.
 *
 * Feature strides must be 1.  A row with no kept key contributes 0; a NaN
 * forward row makes the gradients it touches NaN.  Keys a mask removes are
 * skipped, so a non-finite value stored under a removed key does not reach
 * the gradients.  Kernels: a row-dot kernel for D, then either the tcgen05
 * dK/dV and dQ kernels (see sdpa_bwd_plan) or the general SIMT ones; each
 * output element is written once, so results are deterministic.  Returns SDPA_OK, SDPA_ERR_INVALID (shapes, strides,
 * pointers), SDPA_ERR_UNSUPPORTED (E outside 0..256, Ev outside 1..256, not an sm_100
 * device), SDPA_ERR_WORKSPACE or SDPA_ERR_CUDA.
 */
int sdpa_bwd(const void* q, const void* k, const void* v, const void* out, const float* lse,
             const void* dout, void* dq, void* dk, void* dv,
             int B, int Hq, int Hkv, int L, int S, int E, int Ev,
             const int64_t q_stride[4], const int64_t k_stride[4],
             const int64_t v_stride[4], const int64_t o_stride[4],
             const int64_t do_stride[4], const int64_t dq_stride[4],
             const int64_t dk_stride[4], const int64_t dv_stride[4],
             int has_scale, float scale,
             int mask_kind, const int32_t* cu_seqlens, int n_seqs, int max_seqlen,
             const void* bias, const int64_t bias_stride[4],
             int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Which kernels sdpa_bwd() would run for these arguments (no work is done):
 * 1 = the tcgen05/TMA backward (fp16/bf16, E = Ev in {64, 96, 128}, mask
 * none / causal / block-diagonal, TMA-legal strides and 16-byte aligned
 * pointers), 3 = the general SIMT kernels, or a negative sdpa_status for
 * rejected arguments.  The varlen limits (n_seqs, max_seqlen) are not
 * checked here.
 */
int sdpa_bwd_plan(int B, int Hq, int Hkv, int L, int S, int E, int Ev,
                  const int64_t q_stride[4], const int64_t k_stride[4],
                  const int64_t v_stride[4], const int64_t do_stride[4],
                  const int64_t dq_stride[4], const int64_t dk_stride[4],
                  const int64_t dv_stride[4], int mask_kind, int dtype,
                  const void* q, const void* k, const void* v, const void* dout,
                  const void* dq, const void* dk, const void* dv);

/* Size of the fixed device scratch array of sdpa_decode_fwd_noalloc(). */
#define SDPA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * Decode attention that allocates nothing and takes no workspace.  (No
 * counterpart on the pages: it exists for callers, not for the method.)
 *
 * For callers that cannot allocate device memory when they call (a runtime
 * that reserves all its device memory up front, or a plugin interface that
 * passes only inputs and outputs): the same split-S decode and combine
 * kernels as sdpa_fwd(), with their scratch in a 32 MiB array compiled into
 * the library (SDPA_NOALLOC_SCRATCH_BYTES).  That array occupies 32 MiB on
 * every GPU where the library's code is loaded, until the process exits.
 *
 * Arguments are sdpa_fwd()'s without mask, bias or workspace (mask_kind
 * NONE).  Takes only problems the decode kernel takes: fp16/bf16,
 * E = Ev in {64, 128, 256}, (Hq/Hkv)*L <= 8, 16-byte aligned rows; returns
 * SDPA_ERR_UNSUPPORTED otherwise, and SDPA_ERR_WORKSPACE when the problem
 * needs more scratch than SDPA_NOALLOC_SCRATCH_BYTES (the same bytes
 * sdpa_fwd_workspace_size() reports for it).
 *
 * The first call on each device looks up the array's device address with
 * cudaGetSymbolAddress, with that device current; make that first call
 * before any stream capture.  Every call uses the same array, so calls whose
 * kernels can overlap on the GPU (other streams, other host threads) race
 * and must be serialised by the caller.  Nothing in the array needs to be
 * cleared between calls.
 */
int sdpa_decode_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                            int B, int Hq, int Hkv, int L, int S, int E, int Ev,
                            const int64_t q_stride[4], const int64_t k_stride[4],
                            const int64_t v_stride[4], const int64_t o_stride[4],
                            int has_scale, float scale, int dtype, void* stream);

/*
 * Decode attention over a paged key/value cache.
 *
 * Each batch row's keys and values live in fixed-size pages of two shared
 * pools, found through the row's block table, as in paged KV-cache engines
 * (the hourtab.com xFormers retainer post, "Related retainer posts", names
 * them and their failure mode: pages read beyond what a sequence was given,
 * garbage output, no error).  The keys (values) of row b are the first
 * seq_lens[b] tokens of pages block_table[b * max_pages + 0],
 * block_table[b * max_pages + 1], ... taken in table order; the result is the
 * attention of row b's L query rows over them with no mask, as sdpa_fwd()
 * computes it (a row with seq_lens[b] = 0 gets O = 0 and lse = -inf).
 *
 * Arguments:
 * - q (B, Hq, L, E), out (B, Hq, L, Ev), lse (B, Hq, L) float32: as for
 *   sdpa_fwd(), with q_stride / o_stride in (batch, head, row, feature) order.
 * - k_pages, v_pages: the pools, num_pages pages of page_size tokens and Hkv
 *   heads each; kp_stride / vp_stride are element strides in the order
 *   (page, head, token in page, feature), so both (num_pages, page_size,
 *   Hkv, E) and (num_pages, Hkv, page_size, E) pools are described.
 * - block_table: device int32 [B][max_pages], row-major; seq_lens: device
 *   int32 [B].  Both are read on the device, so they may change between
 *   calls recorded in a CUDA graph.
 * - page_size: a power of two from 1 to 65536; max_pages * page_size <= 2^20.
 * - has_scale / scale, dtype, workspace, stream: as for sdpa_fwd(); the
 *   workspace must hold sdpa_decode_paged_workspace_size() bytes.
 *
 * Supported: fp16 / bf16, E = Ev in {64, 128, 256}, (Hq / Hkv) * L <= 8,
 * 16-byte aligned pointers and strides; SDPA_ERR_UNSUPPORTED otherwise.
 * Errors found on the device never fault and never read outside the pools:
 * a table entry outside [0, num_pages) drops that page's tokens and records
 * code 32, a seq_lens entry outside [0, max_pages * page_size] is clamped
 * and records code 31; sdpa_take_device_error() returns the code.
 */
size_t sdpa_decode_paged_workspace_size(int B, int Hq, int Hkv, int L, int E, int Ev, int page_size,
                                        int max_pages, int dtype);
int sdpa_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                      const int32_t* seq_lens, void* out, float* lse, int B, int Hq, int Hkv, int L, int E,
                      int Ev, int num_pages, int page_size, int max_pages, const int64_t q_stride[4],
                      const int64_t kp_stride[4], const int64_t vp_stride[4], const int64_t o_stride[4],
                      int has_scale, float scale, int dtype, void* workspace, size_t workspace_bytes,
                      void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SDPA15_H */
