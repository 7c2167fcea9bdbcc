// fa_lib.cu -- the C ABI declared in include/fa.h: argument checks, TMA tensor maps, kernel launches, status.
// All kernels live in this one translation unit so they share the per-device status word.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "fa.h"
#include "fa_abi_checks.h"
#include "fa_common.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd256.cuh"
#include "fa_bwd.cuh"
#include "fa_bwd256.cuh"
#include "fa_mask.cuh"

// The device error codes are the fa_status values the host returns for them.
static_assert((int)fa::kDevTimeout == (int)FA_ERR_TIMEOUT && (int)fa::kDevBounds == (int)FA_ERR_BOUNDS,
              "device error codes");

namespace {

constexpr int kVersion = 10300;  // 1.3.0: head dims 32 and 96, per-head block masks
constexpr int kMaxN = 1 << 20;
constexpr long long kMaxElems = 1LL << 34;

thread_local std::string t_last_error;
thread_local cudaEvent_t t_events[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};  // [kernel][start, stop]

// Records the caller's event (if any) for `kernel` on stream `st`.
cudaError_t mark(int kernel, int which, cudaStream_t st) {
  cudaEvent_t e = t_events[kernel][which];
  return e ? cudaEventRecord(e, st) : cudaSuccess;
}
std::atomic<uint64_t> g_budget_ns{2000000000ull};
std::atomic<int> g_fwd_tiles{0};  // Q tiles per forward CTA: 0 = choose per call, 1 or 2 = forced

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Head dims: 64, 128 and 256 natively; 32 and 96 run on the 64 / 128 kernels, whose TMA boxes are 64 columns wide
// and zero-fill the columns past the tensor's own, so the extra columns add nothing to any product.  d = 256 has
// its own forward (fa_fwd256.cuh) and backward (fa_bwd256.cuh) kernels.
bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 96 || d == 128 || d == 256; }
bool fwd_head_dim_ok(int d) { return head_dim_ok(d); }

int cuda_fail(cudaError_t e) {
  t_last_error = cudaGetErrorString(e);
  return FA_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Shape/pointer checks shared by every attention entry point.
int check_common(const void* q, const void* k, const void* v, int B, int H, int N, int d, float scale, int dtype,
                 bool fwd = false) {
  if (!q || !k || !v) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16)) return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || N < 1 || N > kMaxN) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (!(fwd ? fwd_head_dim_ok(d) : head_dim_ok(d))) return FA_ERR_UNSUPPORTED;
  if ((long long)B * H * N * d > kMaxElems) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

// [B*H, N, d] view of a [B, H, N, d] tensor: rows past N of a head are out of bounds (zero-filled by TMA),
// so a ragged last tile never reads the next head.  Box: `box_rows` rows (128, or 32 for the d = 256 V chunks) x
// 64 columns (128 bytes), 128-byte swizzle.
int make_map(CUtensorMap* m, const void* ptr, int BH, int N, int d, int dtype, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    t_last_error = "cuTensorMapEncodeTiled unavailable";
    return FA_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                   const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_error = "cuTensorMapEncodeTiled failed with CUresult " + std::to_string((int)r);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

// {d, H, total} view of a packed [total, H, d] tensor with a {64, 1, 128} box: 128 consecutive tokens of one head,
// 64 columns (128 bytes), 128-byte swizzle -- the same shared-memory image as the dense box.  Tokens past `total`
// read as zero.
int make_map_packed(CUtensorMap* m, const void* ptr, int total, int H, int d, int dtype, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    t_last_error = "cuTensorMapEncodeTiled unavailable";
    return FA_ERR_CUDA;
  }
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)total};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)box_rows};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, dtype == FA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                   const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_error = "cuTensorMapEncodeTiled (packed) failed with CUresult " + std::to_string((int)r);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

// 2-D fp32 view {cols, rows} of the dQ accumulator for TMA reduce-add: box 32 columns (128 bytes) x 32 rows,
// 128-byte swizzle (matches the drain warps' staging layout).
int make_map_f32(CUtensorMap* m, void* ptr, long long rows, int cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    t_last_error = "cuTensorMapEncodeTiled unavailable";
    return FA_ERR_CUDA;
  }
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, ptr, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_error = "cuTensorMapEncodeTiled (fp32) failed with CUresult " + std::to_string((int)r);
    return FA_ERR_CUDA;
  }
  return FA_OK;
}

// cudaFuncSetAttribute for the dynamic shared memory size, once per (kernel, device).  `done_mask` must be a
// distinct object per kernel (kernels of identical signature would otherwise share one cache).
template <typename Kernel>
cudaError_t ensure_smem(Kernel kernel, int bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done_mask.load() & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done_mask.fetch_or(bit);
  return e;
}

template <int D, bool BF, int T, int P>
cudaError_t launch_fwd_k(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, fa::FwdArgs a,
                         cudaStream_t st) {
  using C = fa::FwdCfg<D, T>;
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem(fa::fwd_kernel<D, BF, T, P>, C::kSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  a.npairs = (a.nT + T - 1) / T;  // work units (groups of T Q tiles) per (b, h)
  // persistent: as many CTAs as fit at once (3 - T per SM), each walking its share of the units
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = fa::device_sm_count(dev, &sms)) != cudaSuccess) return e;
  const long long units = (long long)a.BH * a.npairs * (P == fa::kModeSplit ? a.nsplit : 1);
  const unsigned grid = (unsigned)std::min<long long>(units, (long long)sms * (3 - T));
  if ((e = mark(FA_KERNEL_FWD, 0, st)) != cudaSuccess) return e;
  fa::fwd_kernel<D, BF, T, P><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return mark(FA_KERNEL_FWD, 1, st);
}

template <int D, bool BF, int T>
cudaError_t launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdArgs& a,
                       cudaStream_t st) {
  return a.cu_q ? launch_fwd_k<D, BF, T, fa::kModePacked>(mq, mk, mv, a, st)
                : launch_fwd_k<D, BF, T, fa::kModeDense>(mq, mk, mv, a, st);
}

// d = 256: one CTA per SM, persistent over single Q tiles (see Fwd256Cfg).
template <bool BF, int P>
cudaError_t launch_fwd256(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, fa::FwdArgs a,
                          cudaStream_t st) {
  using C = fa::Fwd256Cfg;
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t e = ensure_smem(fa::fwd256_kernel<BF, P>, C::kSmemBytes, smem_set);
  if (e != cudaSuccess) return e;
  a.npairs = a.nT;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = fa::device_sm_count(dev, &sms)) != cudaSuccess) return e;
  const long long units = (long long)a.BH * a.npairs * (P == fa::kModeSplit ? a.nsplit : 1);
  const unsigned grid = (unsigned)std::min<long long>(units, (long long)sms);
  if ((e = mark(FA_KERNEL_FWD, 0, st)) != cudaSuccess) return e;
  fa::fwd256_kernel<BF, P><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return mark(FA_KERNEL_FWD, 1, st);
}

// Q tiles per forward CTA for this call (see FwdCfg).  Measured on B200 (bf16, causal): d = 64 prefers one-tile
// CTAs (GPT-2 shape 273 vs 242 TFLOP/s, BERT shape 203 vs 188), d = 128 two-tile CTAs (N = 4096/8192/16384:
// 763/973/1094 vs 671/930/1034).
int fwd_tiles_for(int d) {
  const int forced = g_fwd_tiles.load();
  if (forced == 1 || forced == 2) return forced;
  return d <= 64 ? 1 : 2;
}

// Packed variable-length batch description (all null / zero for the dense [B, H, N, d] layout).
struct Packed {
  const int32_t* cu_q = nullptr;
  const int32_t* cu_k = nullptr;
  int total_q = 0, total_k = 0, Nk = 0;
};

int run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
            float scale, int causal, const int32_t* key_lens, const int32_t* row_ptr, const int32_t* col_idx,
            int dtype, cudaStream_t st, const Packed& pk = Packed(), long long list_head_stride = 0) {
  CUtensorMap mq, mk, mv;
  int rc;
  const int v_rows = d == 256 ? 32 : 128;  // d = 256 streams V in chunks of 32 keys
  if (pk.cu_q) {
    if ((rc = make_map_packed(&mq, q, pk.total_q, H, d, dtype)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mk, k, pk.total_k, H, d, dtype)) != FA_OK) return rc;
    if ((rc = make_map_packed(&mv, v, pk.total_k, H, d, dtype, v_rows)) != FA_OK) return rc;
  } else {
    if ((rc = make_map(&mq, q, B * H, N, d, dtype)) != FA_OK) return rc;
    if ((rc = make_map(&mk, k, B * H, N, d, dtype)) != FA_OK) return rc;
    if ((rc = make_map(&mv, v, B * H, N, d, dtype, v_rows)) != FA_OK) return rc;
  }
  fa::FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.key_lens = key_lens;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.list_head_stride = list_head_stride;
  a.cu_q = pk.cu_q;
  a.cu_k = pk.cu_k;
  a.total_q = pk.total_q;
  a.total_k = pk.total_k;
  a.Nk = pk.cu_q ? pk.Nk : N;
  a.dl = d;
  a.nsplit = 1;
  a.kv_split_tiles = 0;
  a.o_part = nullptr;
  a.lse_part = nullptr;
  a.H = H;
  a.N = N;
  a.nT = (N + fa::kTile - 1) / fa::kTile;
  a.npairs = (a.nT + 1) / 2;
  a.BH = B * H;
  a.causal = causal ? 1 : 0;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.budget_ns = g_budget_ns.load();
  cudaError_t e;
  const bool bf = dtype == FA_BF16;
  if (d == 256) {
    if (pk.cu_q)
      e = bf ? launch_fwd256<true, fa::kModePacked>(mq, mk, mv, a, st)
             : launch_fwd256<false, fa::kModePacked>(mq, mk, mv, a, st);
    else
      e = bf ? launch_fwd256<true, fa::kModeDense>(mq, mk, mv, a, st)
             : launch_fwd256<false, fa::kModeDense>(mq, mk, mv, a, st);
  } else if (fwd_tiles_for(d) == 2) {
    if (d <= 64)
      e = bf ? launch_fwd<64, true, 2>(mq, mk, mv, a, st) : launch_fwd<64, false, 2>(mq, mk, mv, a, st);
    else
      e = bf ? launch_fwd<128, true, 2>(mq, mk, mv, a, st) : launch_fwd<128, false, 2>(mq, mk, mv, a, st);
  } else {
    if (d <= 64)
      e = bf ? launch_fwd<64, true, 1>(mq, mk, mv, a, st) : launch_fwd<64, false, 1>(mq, mk, mv, a, st);
    else
      e = bf ? launch_fwd<128, true, 1>(mq, mk, mv, a, st) : launch_fwd<128, false, 1>(mq, mk, mv, a, st);
  }
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t lists_bytes(int nT) {
  // row_ptr, col_ptr [nT+1] and col_idx, row_idx [nT*nT], each 256-byte aligned
  return 2 * align_up((size_t)(nT + 1) * 4, 256) + 2 * align_up((size_t)nT * nT * 4, 256);
}

struct Lists {
  int32_t *row_ptr, *col_idx, *col_ptr, *row_idx;
};

Lists carve_lists(void* ws, int nT) {
  uint8_t* p = static_cast<uint8_t*>(ws);
  Lists l;
  l.row_ptr = reinterpret_cast<int32_t*>(p);
  p += align_up((size_t)(nT + 1) * 4, 256);
  l.col_ptr = reinterpret_cast<int32_t*>(p);
  p += align_up((size_t)(nT + 1) * 4, 256);
  l.col_idx = reinterpret_cast<int32_t*>(p);
  p += align_up((size_t)nT * nT * 4, 256);
  l.row_idx = reinterpret_cast<int32_t*>(p);
  return l;
}

// Tile lists of `heads` masks ([heads][nT][nT]); head h's lists are lists_bytes(nT) bytes after head 0's.
int launch_lists(const uint8_t* mask, int nT, const Lists& l, cudaStream_t st, int heads = 1) {
  const long long stride = heads > 1 ? (long long)(lists_bytes(nT) / 4) : 0;
  const int row_blocks = (nT + fa::kMaskWarps - 1) / fa::kMaskWarps;
  const int col_blocks = (nT + 32 * fa::kMaskWarps - 1) / (32 * fa::kMaskWarps);
  const dim3 grid(row_blocks + col_blocks, heads);
  fa::blockmask_count_kernel<<<grid, fa::kMaskWarps * 32, 0, st>>>(mask, nT, l.row_ptr, l.col_ptr, stride);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  fa::blockmask_scan_kernel<<<heads, fa::kMaskThreads, 0, st>>>(nT, l.row_ptr, l.col_ptr, stride);
  if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e);
  fa::blockmask_fill_kernel<<<grid, fa::kMaskWarps * 32, 0, st>>>(mask, nT, l.row_ptr, l.col_idx, l.col_ptr,
                                                                  l.row_idx, stride);
  e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

}  // namespace

// ------------------------------------------------------------------------------------------ split-K/V decode
constexpr int kMaxSplits = 32;

// Splits for a split-K/V forward.  With G persistent CTAs (two one-tile CTAs per SM) and `base` (Q tile, head)
// pairs, s splits take about ceil(base*s / G) rounds of ceil(tiles_k / s) + 1 tile-steps each (one step of per-unit
// overhead); the smallest estimate wins.  Measured on B200 (B8 H16, one query, 16384 keys, d128): 2 splits, one
// round, 5437 GB/s; 3 splits, an uneven second round, 4580 GB/s.
int splitkv_splits(int B, int H, int Nq, int Nk, int requested) {
  const int tiles_k = (Nk + fa::kTile - 1) / fa::kTile;
  if (requested > 0) return std::min(std::min(requested, kMaxSplits), tiles_k);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || fa::device_sm_count(dev, &sms) != cudaSuccess) sms = 148;
  const long long G = 2LL * sms;
  const long long base = (long long)B * H * ((Nq + fa::kTile - 1) / fa::kTile);
  int best = 1;
  long long best_cost = -1;
  for (int s = 1; s <= std::min(kMaxSplits, tiles_k); ++s) {
    const long long rounds = (base * s + G - 1) / G;
    const long long cost = rounds * ((tiles_k + s - 1) / s + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = s;
    }
  }
  return best;
}

// Partial results of a split-K/V forward: O rows as wide as the kernel's head dim (64, 128 or 256), then LSE.
int kernel_dim(int d) { return d <= 64 ? 64 : d <= 128 ? 128 : 256; }

size_t splitkv_bytes(int B, int H, int Nq, int d, int nsplit) {
  const size_t rows = (size_t)nsplit * B * H * ((Nq + fa::kTile - 1) / fa::kTile) * fa::kTile;
  return align_up(rows * kernel_dim(d) * 4, 256) + align_up(rows * 4, 256);
}

template <int D, bool BF>
cudaError_t launch_splitkv(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, fa::FwdArgs a,
                           void* o, float* lse, cudaStream_t st) {
  cudaError_t e;
  if constexpr (D == 256)
    e = launch_fwd256<BF, fa::kModeSplit>(mq, mk, mv, a, st);
  else
    e = launch_fwd_k<D, BF, 1, fa::kModeSplit>(mq, mk, mv, a, st);
  if (e != cudaSuccess) return e;
  const long long rows = (long long)a.BH * a.N;
  const unsigned blocks = (unsigned)std::min<long long>((rows + 7) / 8, 148LL * 16);
  fa::splitkv_combine_kernel<D, BF><<<blocks, 256, 0, st>>>(a.o_part, a.lse_part, o, lse, a.nsplit, a.BH, a.N,
                                                            a.nT * fa::kTile, a.dl);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------ packed batches
int check_packed(const void* q, const void* k, const void* v, const int32_t* cu_q, const int32_t* cu_k, int B, int H,
                 int max_q, int max_k, int total_q, int total_k, int d, float scale, int dtype, bool fwd = false) {
  if (!q || !k || !v || !cu_q || !cu_k) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(cu_q, 4) || !aligned(cu_k, 4))
    return FA_ERR_INVALID_ARG;
  if (B < 1 || H < 1 || max_q < 1 || max_k < 1 || max_q > kMaxN || max_k > kMaxN) return FA_ERR_INVALID_ARG;
  if (total_q < 1 || total_k < 1) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (!(fwd ? fwd_head_dim_ok(d) : head_dim_ok(d))) return FA_ERR_UNSUPPORTED;
  const long long npad = (long long)(max_q + fa::kTile - 1) / fa::kTile * fa::kTile;
  if ((long long)total_q * H * d > kMaxElems || (long long)total_k * H * d > kMaxElems ||
      (long long)B * H * npad * d > kMaxElems)
    return FA_ERR_INVALID_ARG;
  return FA_OK;
}

int fa_abi::bwd_check_args(const void* q, const void* k, const void* v, const void* o, const void* dout,
                           const float* lse, const void* dq, const void* dk, const void* dv, int B, int H, int N, int d,
                           float softmax_scale, const int32_t* key_lens, const uint8_t* block_mask, int dtype) {
  int rc = check_common(q, k, v, B, H, N, d, softmax_scale, dtype);
  if (rc != FA_OK) return rc;
  if (!o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16) || !aligned(dout, 16) || !aligned(lse, 4) || !aligned(dq, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16) || (key_lens && !aligned(key_lens, 4)))
    return FA_ERR_INVALID_ARG;
  const int nT = (N + fa::kTile - 1) / fa::kTile;
  if (block_mask && nT > fa::kMaxMaskTiles) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

extern "C" {

int fa_version(void) { return kVersion; }

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_BOUNDS: return "FA_ERR_BOUNDS";
    default: return "FA_UNKNOWN_STATUS";
  }
}

const char* fa_last_error_string(void) { return t_last_error.c_str(); }

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float softmax_scale, int causal, const int32_t* key_lens, int dtype, void* stream) {
  int rc = check_common(q, k, v, B, H, N, d, softmax_scale, dtype, true);
  if (rc != FA_OK) return rc;
  if (!o || !lse || !aligned(o, 16) || !aligned(lse, 4) || (key_lens && !aligned(key_lens, 4)))
    return FA_ERR_INVALID_ARG;
  return run_fwd(q, k, v, o, lse, B, H, N, d, softmax_scale, causal, key_lens, nullptr, nullptr, dtype,
                 static_cast<cudaStream_t>(stream));
}

size_t fa_blocksparse_workspace_size(int N) {
  if (N < 1 || N > kMaxN) return 0;
  return lists_bytes((N + fa::kTile - 1) / fa::kTile);
}

int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                       float softmax_scale, int causal, const int32_t* key_lens, const uint8_t* block_mask,
                       void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  int rc = check_common(q, k, v, B, H, N, d, softmax_scale, dtype, true);
  if (rc != FA_OK) return rc;
  if (!o || !lse || !block_mask || !aligned(o, 16) || !aligned(lse, 4) || (key_lens && !aligned(key_lens, 4)))
    return FA_ERR_INVALID_ARG;
  const int nT = (N + fa::kTile - 1) / fa::kTile;
  if (nT > fa::kMaxMaskTiles) return FA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < lists_bytes(nT)) return FA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Lists l = carve_lists(workspace, nT);
  if ((rc = launch_lists(block_mask, nT, l, st)) != FA_OK) return rc;
  return run_fwd(q, k, v, o, lse, B, H, N, d, softmax_scale, causal, key_lens, l.row_ptr, l.col_idx, dtype, st);
}

int fa_blockmask_lists(const uint8_t* mask, int nT, int32_t* row_ptr, int32_t* col_idx, int32_t* col_ptr,
                       int32_t* row_idx, void* stream) {
  if (!mask || !row_ptr || !col_idx || !col_ptr || !row_idx || nT < 1 || nT > fa::kMaxMaskTiles)
    return FA_ERR_INVALID_ARG;
  Lists l{row_ptr, col_idx, col_ptr, row_idx};
  return launch_lists(mask, nT, l, static_cast<cudaStream_t>(stream));
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d, int has_block_mask) {
  if (B < 1 || H < 1 || N < 1 || N > kMaxN || !head_dim_ok(d)) return 0;
  if ((long long)B * H * N * d > kMaxElems) return 0;  // B*H stays far below 2^31 after this check
  const int nT = (N + fa::kTile - 1) / fa::kTile;
  return fa::bwd_workspace_bytes(B * H, nT, d) + (has_block_mask ? lists_bytes(nT) : 0);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
           void* dk, void* dv, int B, int H, int N, int d, float softmax_scale, int causal, const int32_t* key_lens,
           const uint8_t* block_mask, void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  int rc = fa_abi::bwd_check_args(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, key_lens, block_mask,
                                  dtype);
  if (rc != FA_OK) return rc;
  const int nT = (N + fa::kTile - 1) / fa::kTile;
  const size_t need = fa_bwd_workspace_size(B, H, N, d, block_mask != nullptr);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int32_t *col_ptr = nullptr, *row_idx = nullptr;
  if (block_mask) {
    const Lists l = carve_lists(static_cast<uint8_t*>(workspace) + fa::bwd_workspace_bytes(B * H, nT, d), nT);
    if ((rc = launch_lists(block_mask, nT, l, st)) != FA_OK) return rc;
    col_ptr = l.col_ptr;
    row_idx = l.row_idx;
  }
  CUtensorMap mq, mk, mv, mdo;
  if ((rc = make_map(&mq, q, B * H, N, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H, N, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H, N, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mdo, dout, B * H, N, d, dtype)) != FA_OK) return rc;
  CUtensorMap mdq;  // the fp32 dQ accumulator sits at the start of the workspace: [B*H*Npad, d]
  if ((rc = make_map_f32(&mdq, workspace, (long long)B * H * nT * fa::kTile, d)) != FA_OK) return rc;
  cudaError_t e = fa::run_bwd(mq, mk, mv, mdo, mdq, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, causal != 0,
                              key_lens, col_ptr, row_idx, workspace, dtype == FA_BF16, g_budget_ns.load(), st,
                              t_events[FA_KERNEL_BWD_MAIN][0], t_events[FA_KERNEL_BWD_MAIN][1]);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* cu_seqlens_q,
                  const int32_t* cu_seqlens_k, int B, int H, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int d, float softmax_scale, int causal, int dtype, void* stream) {
  int rc = check_packed(q, k, v, cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q, max_seqlen_k, total_q, total_k, d,
                        softmax_scale, dtype, true);
  if (rc != FA_OK) return rc;
  if (!o || !lse || !aligned(o, 16) || !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  Packed pk;
  pk.cu_q = cu_seqlens_q;
  pk.cu_k = cu_seqlens_k;
  pk.total_q = total_q;
  pk.total_k = total_k;
  pk.Nk = max_seqlen_k;
  return run_fwd(q, k, v, o, lse, B, H, max_seqlen_q, d, softmax_scale, causal, nullptr, nullptr, nullptr, dtype,
                 static_cast<cudaStream_t>(stream), pk);
}

size_t fa_bwd_varlen_workspace_size(int B, int H, int max_seqlen_q, int d) {
  if (B < 1 || H < 1 || max_seqlen_q < 1 || max_seqlen_q > kMaxN || !head_dim_ok(d)) return 0;
  return fa::bwd_workspace_bytes(B * H, (max_seqlen_q + fa::kTile - 1) / fa::kTile, d);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int H,
                  int max_seqlen_q, int max_seqlen_k, int total_q, int total_k, int d, float softmax_scale, int causal,
                  void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  int rc = check_packed(q, k, v, cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q, max_seqlen_k, total_q, total_k, d,
                        softmax_scale, dtype);
  if (rc != FA_OK) return rc;
  if (!o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16) || !aligned(dout, 16) || !aligned(lse, 4) || !aligned(dq, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16))
    return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_varlen_workspace_size(B, H, max_seqlen_q, d);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if ((rc = make_map_packed(&mq, q, total_q, H, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map_packed(&mk, k, total_k, H, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map_packed(&mv, v, total_k, H, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map_packed(&mdo, dout, total_q, H, d, dtype)) != FA_OK) return rc;
  const int nTq = (max_seqlen_q + fa::kTile - 1) / fa::kTile;
  if ((rc = make_map_f32(&mdq, workspace, (long long)B * H * nTq * fa::kTile, d)) != FA_OK) return rc;
  cudaError_t e = fa::run_bwd(mq, mk, mv, mdo, mdq, o, dout, lse, dq, dk, dv, B, H, max_seqlen_q, d, softmax_scale,
                              causal != 0, nullptr, nullptr, nullptr, workspace, dtype == FA_BF16, g_budget_ns.load(),
                              static_cast<cudaStream_t>(stream), t_events[FA_KERNEL_BWD_MAIN][0],
                              t_events[FA_KERNEL_BWD_MAIN][1], cu_seqlens_q, cu_seqlens_k, total_q, total_k,
                              max_seqlen_k);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

size_t fa_fwd_splitkv_workspace_size(int B, int H, int Nq, int Nk, int d, int num_splits) {
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || Nq > kMaxN || Nk > kMaxN || !fwd_head_dim_ok(d)) return 0;
  if (num_splits < 0 || num_splits > kMaxSplits) return 0;
  return splitkv_bytes(B, H, Nq, d, splitkv_splits(B, H, Nq, Nk, num_splits));
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
                   int d, float softmax_scale, int causal, const int32_t* key_lens, int num_splits, void* workspace,
                   size_t workspace_bytes, int dtype, void* stream) {
  int rc = check_common(q, k, v, B, H, Nk, d, softmax_scale, dtype, true);
  if (rc != FA_OK) return rc;
  if (Nq < 1 || Nq > kMaxN || (long long)B * H * Nq * d > kMaxElems) return FA_ERR_INVALID_ARG;
  if (num_splits < 0 || num_splits > kMaxSplits) return FA_ERR_INVALID_ARG;
  if (!o || !lse || !aligned(o, 16) || !aligned(lse, 4) || (key_lens && !aligned(key_lens, 4)))
    return FA_ERR_INVALID_ARG;
  const int nsplit = splitkv_splits(B, H, Nq, Nk, num_splits);
  const size_t need = splitkv_bytes(B, H, Nq, d, nsplit);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  CUtensorMap mq, mk, mv;
  if ((rc = make_map(&mq, q, B * H, Nq, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H, Nk, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H, Nk, d, dtype, d == 256 ? 32 : 128)) != FA_OK) return rc;
  fa::FwdArgs a;
  a.o = o;
  a.lse = lse;
  a.key_lens = key_lens;
  a.row_ptr = nullptr;
  a.col_idx = nullptr;
  a.list_head_stride = 0;
  a.cu_q = nullptr;
  a.cu_k = nullptr;
  a.total_q = 0;
  a.total_k = 0;
  a.H = H;
  a.N = Nq;
  a.Nk = Nk;
  a.dl = d;
  a.nT = (Nq + fa::kTile - 1) / fa::kTile;
  a.npairs = a.nT;  // one Q tile per CTA
  a.BH = B * H;
  a.causal = causal ? 1 : 0;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.budget_ns = g_budget_ns.load();
  const int tiles_k = (Nk + fa::kTile - 1) / fa::kTile;
  a.nsplit = nsplit;
  a.kv_split_tiles = (tiles_k + nsplit - 1) / nsplit;
  const size_t rows = (size_t)nsplit * a.BH * a.nT * fa::kTile;
  a.o_part = static_cast<float*>(workspace);
  a.lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + align_up(rows * kernel_dim(d) * 4, 256));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool bf = dtype == FA_BF16;
  cudaError_t e;
  if (d <= 64)
    e = bf ? launch_splitkv<64, true>(mq, mk, mv, a, o, lse, st) : launch_splitkv<64, false>(mq, mk, mv, a, o, lse, st);
  else if (d <= 128)
    e = bf ? launch_splitkv<128, true>(mq, mk, mv, a, o, lse, st)
           : launch_splitkv<128, false>(mq, mk, mv, a, o, lse, st);
  else
    e = bf ? launch_splitkv<256, true>(mq, mk, mv, a, o, lse, st)
           : launch_splitkv<256, false>(mq, mk, mv, a, o, lse, st);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

size_t fa_blocksparse_heads_workspace_size(int H, int N) {
  if (H < 1 || N < 1 || N > kMaxN) return 0;
  return (size_t)H * lists_bytes((N + fa::kTile - 1) / fa::kTile);
}

int fa_fwd_blocksparse_heads(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                             int d, float softmax_scale, int causal, const int32_t* key_lens,
                             const uint8_t* block_masks, void* workspace, size_t workspace_bytes, int dtype,
                             void* stream) {
  int rc = check_common(q, k, v, B, H, N, d, softmax_scale, dtype, true);
  if (rc != FA_OK) return rc;
  if (!o || !lse || !block_masks || !aligned(o, 16) || !aligned(lse, 4) || (key_lens && !aligned(key_lens, 4)))
    return FA_ERR_INVALID_ARG;
  const int nT = (N + fa::kTile - 1) / fa::kTile;
  if (nT > fa::kMaxMaskTiles) return FA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < fa_blocksparse_heads_workspace_size(H, N))
    return FA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Lists l = carve_lists(workspace, nT);
  if ((rc = launch_lists(block_masks, nT, l, st, H)) != FA_OK) return rc;
  return run_fwd(q, k, v, o, lse, B, H, N, d, softmax_scale, causal, key_lens, l.row_ptr, l.col_idx, dtype, st,
                 Packed(), H > 1 ? (long long)(lists_bytes(nT) / 4) : 0);
}

size_t fa_bwd_blocksparse_heads_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || N > kMaxN || !head_dim_ok(d)) return 0;
  const int nT = (N + fa::kTile - 1) / fa::kTile;
  return fa::bwd_workspace_bytes(B * H, nT, d) + (size_t)H * lists_bytes(nT);
}

int fa_bwd_blocksparse_heads(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                             float softmax_scale, int causal, const int32_t* key_lens, const uint8_t* block_masks,
                             void* workspace, size_t workspace_bytes, int dtype, void* stream) {
  int rc = check_common(q, k, v, B, H, N, d, softmax_scale, dtype);
  if (rc != FA_OK) return rc;
  if (!o || !dout || !lse || !dq || !dk || !dv || !block_masks) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16) || !aligned(dout, 16) || !aligned(lse, 4) || !aligned(dq, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16) || (key_lens && !aligned(key_lens, 4)))
    return FA_ERR_INVALID_ARG;
  const int nT = (N + fa::kTile - 1) / fa::kTile;
  if (nT > fa::kMaxMaskTiles) return FA_ERR_INVALID_ARG;
  const size_t need = fa_bwd_blocksparse_heads_workspace_size(B, H, N, d);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < need) return FA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Lists l = carve_lists(static_cast<uint8_t*>(workspace) + fa::bwd_workspace_bytes(B * H, nT, d), nT);
  if ((rc = launch_lists(block_masks, nT, l, st, H)) != FA_OK) return rc;
  CUtensorMap mq, mk, mv, mdo, mdq;
  if ((rc = make_map(&mq, q, B * H, N, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mk, k, B * H, N, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mv, v, B * H, N, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map(&mdo, dout, B * H, N, d, dtype)) != FA_OK) return rc;
  if ((rc = make_map_f32(&mdq, workspace, (long long)B * H * nT * fa::kTile, d)) != FA_OK) return rc;
  cudaError_t e = fa::run_bwd(mq, mk, mv, mdo, mdq, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, causal != 0,
                              key_lens, l.col_ptr, l.row_idx, workspace, dtype == FA_BF16, g_budget_ns.load(), st,
                              t_events[FA_KERNEL_BWD_MAIN][0], t_events[FA_KERNEL_BWD_MAIN][1], nullptr, nullptr, 0, 0,
                              0, H > 1 ? (long long)(lists_bytes(nT) / 4) : 0);
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_last_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(fa::g_device_status, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return v == 0 ? FA_OK : v;
}

int fa_set_wait_budget_ns(uint64_t budget_ns) {
  if (budget_ns < 1000) return FA_ERR_INVALID_ARG;
  g_budget_ns.store(budget_ns);
  return FA_OK;
}

int fa_set_kernel_events(int kernel, void* start_event, void* stop_event) {
  if (kernel != FA_KERNEL_FWD && kernel != FA_KERNEL_BWD_MAIN) return FA_ERR_INVALID_ARG;
  if ((start_event == nullptr) != (stop_event == nullptr)) return FA_ERR_INVALID_ARG;
  t_events[kernel][0] = static_cast<cudaEvent_t>(start_event);
  t_events[kernel][1] = static_cast<cudaEvent_t>(stop_event);
  return FA_OK;
}

int fa_set_fwd_tiles_per_cta(int tiles) {
  if (tiles < 0 || tiles > 2) return FA_ERR_INVALID_ARG;
  g_fwd_tiles.store(tiles);
  return FA_OK;
}

int fa_debug_build(void) { return FA_DEBUG ? 1 : 0; }

int fa_last_bounds_site(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return -cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, fa::g_bounds_site, sizeof(int));
  if (e != cudaSuccess) return -cuda_fail(e);
  if (v != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(fa::g_bounds_site, &zero, sizeof(int));
    if (e != cudaSuccess) return -cuda_fail(e);
  }
  return v;
}

int fa_selftest_bounds(void* stream) {
  fa::selftest_bounds_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>();
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_selftest_exp2(const float* x, float* out_fma, float* out_mufu, int n, void* stream) {
  if (!x || !out_fma || !out_mufu || n < 1) return FA_ERR_INVALID_ARG;
  const int blocks = (n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024;
  fa::selftest_exp2_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, out_fma, out_mufu, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_selftest_wait_timeout(uint64_t budget_ns, void* stream) {
  if (budget_ns < 1000 || budget_ns > 1000000000ull) return FA_ERR_INVALID_ARG;
  fa::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(budget_ns);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

}  // extern "C"
