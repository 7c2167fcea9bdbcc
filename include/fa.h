/*
 * fa.h -- C ABI of libfa.so: exact IO-aware attention (tiled forward with online softmax, backward by
 * recomputation, optional 128x128 block-sparse tile mask) for NVIDIA B200 (sm_100a).
 *
 * What the library computes (FlashAttention review page, "Method" and claim C2: exact attention, only the output
 * and a small normalisation state written to HBM; claim C7: backward recomputes tiles from the saved state;
 * explainer page, "standard attention", "online softmax" and block-sparse sections):
 *     S = softmax_scale * Q K^T with masked entries at -inf,  P = softmax(S) per row,  O = P V,
 *     LSE_r = log sum_c exp(S_rc)   (natural log; -inf for a row with no visible key, whose O row is 0),
 *     and for the loss sum(O * dO):  D = rowsum(dO * O),  dV = P^T dO,  dS = P * (dO V^T - D),
 *     dQ = softmax_scale * dS K,  dK = softmax_scale * dS^T Q.
 * Key c is visible from query row r of sequence b iff (causal == 0 || c <= r) && (key_lens == NULL ||
 * c < key_lens[b]) && (block_mask == NULL || block_mask[(r/128)*nT + c/128] != 0).
 *
 * Conventions shared by every call
 *   Layout      q, k, v, o, dO, dq, dk, dv: [B, H, N, d] contiguous, d innermost, 16-bit (dtype below).
 *               lse: [B, H, N] fp32.  key_lens: [B] int32 with 0 <= key_lens[b] <= N.
 *               block_mask: [nT, nT] uint8 (0 = skip tile), nT = ceil(N/128), shared by all b and h.
 *   Pointers    Device pointers, 16-byte aligned, caller-owned; the library never allocates, frees or keeps them.
 *               Scratch that a call needs is passed in as `workspace` (device memory, 256-byte aligned) of at
 *               least the size returned by the matching *_workspace_size query.
 *   Shapes      B >= 1, H >= 1, 1 <= N <= 1048576 (2^20), d in {32, 64, 96, 128, 256} (32 and 96 run on the 64
 *               and 128 kernels with the extra columns zero, at their cost; 256 has its own forward and backward
 *               kernels), for every call.  B*H*N*d <= 2^34, softmax_scale finite and > 0.
 *   Execution   Asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).  Inputs must stay valid
 *               until the stream reaches the work.
 *   Errors      Argument errors are detected on the host before anything is launched and returned as an
 *               fa_status; launch failures return FA_ERR_CUDA.  Errors found by the kernels while running (a
 *               pipeline wait that exceeded its time budget; in the debug build also a failed index check) are
 *               recorded in a per-device status word and returned by fa_last_device_status().  Non-finite inputs
 *               are not checked; they propagate.
 *   Debug build libfa_debug.so (same entry points, compiled with FA_DEBUG=1) checks every index its kernels
 *               compute for a global-memory access against the extent of the buffer it addresses; a failed check
 *               skips that access and records FA_ERR_BOUNDS plus a site code (fa_last_bounds_site).
 *   Threads     Calls may come from several host threads; each call only reads library state that is set once.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad shape, scale <= 0, bad dtype */
  FA_ERR_UNSUPPORTED = 2, /* head dimension other than 32, 64, 96, 128, 256 */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (message: fa_last_error_string) */
  FA_ERR_TIMEOUT = 4,     /* a kernel wait ran out of its time budget (device-detected) */
  FA_ERR_WORKSPACE = 5,   /* workspace missing, misaligned or smaller than the query says */
  FA_ERR_BOUNDS = 6       /* debug build only: a kernel's index check failed and the access was skipped */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/* Library version as major*10000 + minor*100 + patch. */
int fa_version(void);

/* Human-readable name of an fa_status value (static string). */
const char* fa_status_string(int status);

/* Text of the last CUDA error seen by a call on this host thread ("" if none). */
const char* fa_last_error_string(void);

/*
 * Forward (review page "Method"; slide deck "Executable shape"): persistent CTAs each take 128-row Q tiles (two
 * tiles that alternate on the tensor core per CTA at d = 96 / 128, one tile per CTA and two CTAs per SM at d <= 64,
 * one tile per CTA at d = 256), stream the visible 128-key K/V tiles through shared memory, keep the running max
 * and denominator per row on chip and write only O and LSE.  Tiles that the causal mask or the key lengths hide
 * entirely are never loaded.
 *   q, k, v   in   [B,H,N,d]     o   out [B,H,N,d]     lse  out [B,H,N] fp32 (natural log)
 *   causal    nonzero: key c visible from row r only if c <= r
 *   key_lens  optional [B] int32 device array (NULL: every key visible)
 *   dtype     fa_dtype of q, k, v and o
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float softmax_scale, int causal, const int32_t* key_lens, int dtype, void* stream);

/* Bytes of workspace fa_fwd_blocksparse needs for sequence length N (the tile lists). */
size_t fa_blocksparse_workspace_size(int N);

/*
 * Block-sparse forward (explainer page, block-sparse section: masking whole tiles means never loading them).
 * Same arguments as fa_fwd plus a device block_mask [nT*nT] uint8.  The call first converts the mask into
 * per-row lists of kept tiles in `workspace` (device kernel), then runs the forward over those lists only;
 * causal and key_lens still apply inside kept tiles.  The result is exact attention under the combined mask.
 */
int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                       int d, float softmax_scale, int causal, const int32_t* key_lens, const uint8_t* block_mask,
                       void* workspace, size_t workspace_bytes, int dtype, void* stream);

/* Bytes of workspace fa_bwd needs (fp32 dQ accumulator, per-row LSE and D terms, tile lists if masked). */
size_t fa_bwd_workspace_size(int B, int H, int N, int d, int has_block_mask);

/*
 * Backward (review page claim C7: P is recomputed tile by tile from the saved LSE; the N x N matrix never exists
 * in HBM).  Inputs q, k, v, o, dO [B,H,N,d] and lse [B,H,N] from fa_fwd with the same mask arguments; outputs
 * dq, dk, dv [B,H,N,d] (fully overwritten).  block_mask may be NULL.  Runs a preprocessing kernel (D = rowsum(dO*O),
 * zeroed dQ accumulator), the main kernel (persistent CTAs, each walking 128-key tiles and, per tile, the visible
 * Q tiles; dK, dV accumulate on chip, dQ partial sums go into the fp32 accumulator in the workspace by bulk
 * reduce-add) and a conversion kernel for dQ.  At d = 256 the main kernel makes two passes per 128-key tile, one
 * per half of the head dimension (each recomputes the scores over the full d and produces that half of dK, dV
 * and dQ), because one pass's dK and dV would not fit the tensor memory.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, int B, int H, int N, int d, float softmax_scale, int causal,
           const int32_t* key_lens, const uint8_t* block_mask, void* workspace, size_t workspace_bytes, int dtype,
           void* stream);

/*
 * Block-mask index lists on the device (explainer page, block-sparse section), exposed for exact checks:
 * from mask [nT*nT] uint8 builds CSR row_ptr [nT+1] / col_idx [nT*nT] (kept tiles per row, ascending) and CSC
 * col_ptr [nT+1] / row_idx [nT*nT] (kept tiles per column, ascending).  All pointers are device pointers;
 * 1 <= nT <= 8192.
 */
int fa_blockmask_lists(const uint8_t* mask, int nT, int32_t* row_ptr, int32_t* col_idx, int32_t* col_ptr,
                       int32_t* row_idx, void* stream);

/*
 * Per-head block masks: as fa_fwd_blocksparse / fa_bwd, but block_masks is [H, nT, nT] uint8 (head h's mask at
 * block_masks + h*nT*nT, shared by all b).  The pages describe one tile mask; a separate mask per head is the same
 * tile skipping with one CSR/CSC list set per head (explainer page, block-sparse section).  Workspace:
 * fa_blocksparse_heads_workspace_size(H, N) for the forward, fa_bwd_blocksparse_heads_workspace_size(B, H, N, d)
 * for the backward.
 */
size_t fa_blocksparse_heads_workspace_size(int H, int N);

int fa_fwd_blocksparse_heads(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                             int d, float softmax_scale, int causal, const int32_t* key_lens,
                             const uint8_t* block_masks, void* workspace, size_t workspace_bytes, int dtype,
                             void* stream);

size_t fa_bwd_blocksparse_heads_workspace_size(int B, int H, int N, int d);

int fa_bwd_blocksparse_heads(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                             float softmax_scale, int causal, const int32_t* key_lens, const uint8_t* block_masks,
                             void* workspace, size_t workspace_bytes, int dtype, void* stream);

/*
 * Packed variable-length batches.  The pages give no interface for this (it generalises the key-length masking
 * they describe for padded BERT batches, explainer page, block-sparse and masking section): B sequences of
 * different lengths are stored back to back without padding.
 *   Layout      q, o, dO, dq: [total_q, H, d]; k, v, dk, dv: [total_k, H, d] (token-major, d innermost, 16-bit);
 *               lse: [H, total_q] fp32 (natural log, -inf for a row with no visible key).
 *               cu_seqlens_q [B+1], cu_seqlens_k [B+1]: int32 device arrays, cu[0] = 0, non-decreasing,
 *               cu[B] = total; sequence b is tokens cu[b] .. cu[b+1]-1.  len_q(b) <= max_seqlen_q and
 *               len_k(b) <= max_seqlen_k (both <= 2^20).  Values outside these rules are clamped into range on the
 *               device (no access leaves the tensors) but the results for such sequences are unspecified.
 *   Visibility  Key c of sequence b is visible from its query r (positions within the sequence) iff
 *               c < len_k(b) && (causal == 0 || c <= r).  For len_q == len_k this is ordinary causal self-attention.
 *   Shapes      total_q, total_k >= 1; total*H*d and B*H*ceil(max_seqlen_q/128)*128*d <= 2^34; d as for fa_fwd.
 * Everything else (pointers, execution, errors) is as for fa_fwd / fa_bwd.  No block mask, no key_lens.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                  const int32_t* cu_seqlens_k, int B, int H, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int d, float softmax_scale, int causal, int dtype, void* stream);

/*
 * Split-K/V forward for decoding: a few new queries per (b, h) against a long key/value cache.  The pages give no
 * interface for this (they note the kernel's central role in inference and keeping K/V resident, review page,
 * "Impact"); it reuses the tiled forward with the keys cut into ranges processed in parallel, each range's
 * normalised O and LSE kept in fp32, and a merge of the ranges by their LSE (the online-softmax rescaling of the
 * explainer page applied to whole partial results).
 *   Layout      q, o: [B, H, Nq, d]; k, v: [B, H, Nk, d] (16-bit, d innermost); lse: [B, H, Nq] fp32 natural log.
 *               key_lens: optional [B] int32, the number of valid cache entries of sequence b (<= Nk).
 *   Visibility  The Nq queries are the last Nq positions of their sequence: with len = key_lens[b] (or Nk), key c
 *               is visible from query r iff c < len && (causal == 0 || c <= r + len - Nq).  (This differs from
 *               fa_fwd's causal, which aligns query and key 0.)  A query with no visible key gets O = 0, LSE = -inf.
 *   Splits      num_splits in [0, 32]; 0 picks enough ranges to fill the GPU.  The result does not depend on the
 *               number of splits beyond fp32 rounding.
 *   Workspace   fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, num_splits) bytes (256-byte aligned device memory).
 *   Shapes      1 <= Nq, Nk <= 2^20, B*H*Nq*d and B*H*Nk*d <= 2^34, d as for fa_fwd.  Everything else as fa_fwd.
 */
size_t fa_fwd_splitkv_workspace_size(int B, int H, int Nq, int Nk, int d, int num_splits);

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                   int d, float softmax_scale, int causal, const int32_t* key_lens, int num_splits, void* workspace,
                   size_t workspace_bytes, int dtype, void* stream);

/* Bytes of workspace fa_bwd_varlen needs (fp32 dQ accumulator and per-row LSE/D over B*H padded sequences). */
size_t fa_bwd_varlen_workspace_size(int B, int H, int max_seqlen_q, int d);

/* Backward of fa_fwd_varlen: dq [total_q,H,d], dk, dv [total_k,H,d] (fully overwritten); same kernels as fa_bwd. */
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int H,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int d, float softmax_scale, int causal,
                  void* workspace, size_t workspace_bytes, int dtype, void* stream);

/*
 * Synchronises `stream`, then returns and clears the current device's status word: FA_OK, or FA_ERR_TIMEOUT if a
 * kernel abandoned a wait since the last query (its outputs are then unspecified).  FA_ERR_CUDA if the
 * synchronisation itself failed.
 */
int fa_last_device_status(void* stream);

/*
 * Time budget of every pipeline wait inside the kernels, in nanoseconds (default 2e9).  A wait that exceeds it
 * records FA_ERR_TIMEOUT and the kernel unwinds (drains its own copies, frees its tensor memory, returns).
 * Values below 1000 are rejected with FA_ERR_INVALID_ARG.  Process-wide; affects launches made after the call.
 */
int fa_set_wait_budget_ns(uint64_t budget_ns);

/*
 * Self-test of the timeout path: launches one CTA that waits on an mbarrier nobody arrives on, with the given
 * budget (1000 ns .. 1e9 ns).  The wait gives up, records FA_ERR_TIMEOUT in the status word and the kernel returns
 * normally; read the result with fa_last_device_status().
 */
int fa_selftest_wait_timeout(uint64_t budget_ns, void* stream);

/*
 * Tuning override (no counterpart in the paper): number of 128-row Q tiles one forward CTA owns.  2 = one CTA per
 * SM whose two tiles alternate on the tensor core; 1 = two one-tile CTAs per SM (finer scheduling); 0 (default) =
 * chosen per call.  Results are identical up to rounding order.  Process-wide; FA_ERR_INVALID_ARG outside 0..2.
 */
int fa_set_fwd_tiles_per_cta(int tiles);

/*
 * Self-test of the forward's FMA-pipe exponential (no counterpart in the paper): for n device floats x, writes the
 * library's range-reduced polynomial 2^x to out_fma and the hardware ex2.approx result to out_mufu (device
 * pointers, caller-owned).  Used by the tests to bound the polynomial's relative error.
 */
int fa_selftest_exp2(const float* x, float* out_fma, float* out_mufu, int n, void* stream);

/* 1 if this library is the debug build (index checks compiled in), else 0. */
int fa_debug_build(void);

/*
 * Synchronises `stream`, then returns and clears the site code of the first failed index check since the last
 * query (0 if none; always 0 in the release build).  Sites: 1 forward O row, 2 forward LSE, 3 split-K/V partials,
 * 4 split-K/V combine, 5 d = 256 forward O / LSE, 11 backward per-row side data, 12 backward dQ reduce box,
 * 13 backward dK / dV row, 14 backward preprocess row, 15 dQ conversion, 21 block-mask list entry, 99 self-test.
 * A negative value is an FA_ERR_CUDA from the synchronisation or the read.
 */
int fa_last_bounds_site(void* stream);

/*
 * Self-test of the index checks: one thread stores to a 4-entry device array through the check, at indices 0..4.
 * In the debug build the last one fails its check: FA_ERR_BOUNDS is recorded (fa_last_device_status) with site 99
 * (fa_last_bounds_site) and that store is skipped.  In the release build the checks are compiled out and nothing
 * is recorded.  No access outside the array is made in either build.
 */
int fa_selftest_bounds(void* stream);

/* Size of the fixed device scratch array behind fa_bwd_noalloc: 32 MiB of device memory on every GPU whose context
 * loads the array's module, held until that context is destroyed (normally process exit).  With lazy module loading
 * (the CUDA 12 default) the module is loaded by the first fa_bwd_noalloc call on a device; with eager loading
 * (CUDA_MODULE_LOADING=EAGER) when the context is created, whether or not fa_bwd_noalloc is ever called. */
#define FA_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * fa_bwd without a workspace argument, for callers that cannot allocate device memory when they run the backward
 * (for example code inside a framework or plugin host that owns all device memory and forbids allocation during
 * execution, or a latency-sensitive loop that cannot pay for cudaMalloc's implicit synchronisation).  No
 * counterpart in the paper: it is a packaging of the same computation.  The scratch fa_bwd needs comes from a
 * file-scope device array of FA_NOALLOC_SCRATCH_BYTES inside the library; this call allocates nothing and calls no
 * allocating routine.  Arguments, layouts and results are exactly those of fa_bwd.
 *   Size limit  problems whose fa_bwd_workspace_size() exceeds FA_NOALLOC_SCRATCH_BYTES are rejected with
 *               FA_ERR_WORKSPACE before anything is launched (e.g. B*H = 96, N = 1024, d = 64 needs 24.75 MiB: fits).
 *   Set-up      the first call on a device looks up the array's device address (cudaGetSymbolAddress) with that
 *               device current; make that first call before any stream capture.  The address is cached per device
 *               together with the id of the context it belongs to: after cudaDeviceReset (a new context, in which
 *               the array may have moved) the next call looks it up again, so that call, too, must not be the
 *               first one made inside a capture.
 *   Checks      the same argument checks as fa_bwd, in the same order and with the same status codes; only then
 *               is the size limit applied.
 *   Sharing     every call on a device uses the same array and it keeps the last call's contents (each call
 *               rewrites what it reads, including zeroing its dQ accumulator).  Calls that overlap on the GPU (on
 *               different streams, or from different host threads without ordering) race on the array.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, int B, int H, int N, int d, float softmax_scale, int causal,
                   const int32_t* key_lens, const uint8_t* block_mask, int dtype, void* stream);

/* Kernels that fa_set_kernel_events can bracket. */
typedef enum { FA_KERNEL_FWD = 0, FA_KERNEL_BWD_MAIN = 1 } fa_kernel_id;

/*
 * Measurement hook (no counterpart on the pages): on this host thread, make the next calls record `start_event`
 * immediately before and `stop_event` immediately after the launch of the given kernel (fa_fwd's kernel, or the
 * main kernel of fa_bwd), on the call's stream.  Events are cudaEvent_t handles owned by the caller; NULL for both
 * turns the hook off.  Returns FA_ERR_INVALID_ARG for an unknown kernel id or a half-set pair.
 */
int fa_set_kernel_events(int kernel, void* start_event, void* stop_event);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
