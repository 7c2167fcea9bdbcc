// fa_mask.cuh -- block-mask tile lists on the device (explainer page, block-sparse section: kept tiles are the
// only ones loaded), and the wait-timeout self-test kernel.
#pragma once
#include "fa_common.cuh"

namespace fa {

constexpr int kMaskThreads = 1024;  // threads of the prefix-scan kernel
constexpr int kMaskWarps = 8;       // warps per CTA of the count and fill kernels
constexpr int kMaxMaskTiles = 8192;

// Tile lists of a block mask in three launches, integer only (the result is unique, so it must equal any correct
// CPU construction exactly):
//   blockmask_count_kernel  kept tiles per row (one warp per row, coalesced byte loads and a warp sum) into
//                           row_ptr[i+1], and per column (one warp per strip of 32 columns, lane = column, walking
//                           the rows) into col_ptr[j+1]
//   blockmask_scan_kernel   in-place prefix sums: row_ptr, col_ptr become the CSR / CSC offsets
//   blockmask_fill_kernel   each row's kept columns in ascending order (warp ballot compaction) into col_idx, and
//                           each column's kept rows in ascending order (the strip's lanes walk the rows in order)
//                           into row_idx
// The count and fill kernels take ceil(nT/8) CTAs for rows followed by ceil(nT/256) CTAs for column strips; grid.y
// is the number of masks.  Per-head masks: mask h is at mask + h*nT*nT and its lists `head_stride` int32 further
// on than head 0's (one mask for all heads: grid.y = 1, stride 0).
__device__ __forceinline__ int mask_row_blocks(int nT) { return (nT + kMaskWarps - 1) / kMaskWarps; }

__global__ void __launch_bounds__(kMaskWarps * 32)
    blockmask_count_kernel(const uint8_t* __restrict__ mask, int nT, int32_t* __restrict__ row_ptr,
                           int32_t* __restrict__ col_ptr, long long head_stride) {
  mask += (size_t)blockIdx.y * nT * nT;
  row_ptr += blockIdx.y * head_stride;
  col_ptr += blockIdx.y * head_stride;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int rb = mask_row_blocks(nT);
  if ((int)blockIdx.x < rb) {
    const int i = blockIdx.x * kMaskWarps + warp;
    if (i >= nT) return;
    const uint8_t* r = mask + (size_t)i * nT;
    int c = 0;
    for (int x = lane; x < nT; x += 32) c += r[x] != 0;
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) c += __shfl_xor_sync(0xffffffffu, c, m);
    if (lane == 0) row_ptr[i + 1] = c;
  } else {
    const int j = ((blockIdx.x - rb) * kMaskWarps + warp) * 32 + lane;
    if (j >= nT) return;
    int c = 0;
#pragma unroll 8
    for (int x = 0; x < nT; ++x) c += mask[(size_t)x * nT + j] != 0;
    col_ptr[j + 1] = c;
  }
}

// One CTA per mask: counts at [1, nT] become inclusive prefix sums in place, [0] = 0.
__global__ void __launch_bounds__(kMaskThreads, 1)
    blockmask_scan_kernel(int nT, int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_ptr,
                          long long head_stride) {
  row_ptr += blockIdx.x * head_stride;
  col_ptr += blockIdx.x * head_stride;
  __shared__ int32_t part_r[kMaskThreads], part_c[kMaskThreads];
  const int tid = threadIdx.x;
  // each thread owns a contiguous chunk of the counts
  const int chunk = (nT + kMaskThreads - 1) / kMaskThreads;
  const int lo = tid * chunk, hi = min(lo + chunk, nT);
  int sr = 0, sc = 0;
  for (int i = lo; i < hi; ++i) { sr += row_ptr[i + 1]; sc += col_ptr[i + 1]; }
  part_r[tid] = sr;
  part_c[tid] = sc;
  __syncthreads();
  for (int off = 1; off < kMaskThreads; off <<= 1) {  // inclusive scan of the chunk sums
    const int ar = tid >= off ? part_r[tid - off] : 0;
    const int ac = tid >= off ? part_c[tid - off] : 0;
    __syncthreads();
    part_r[tid] += ar;
    part_c[tid] += ac;
    __syncthreads();
  }
  int run_r = part_r[tid] - sr, run_c = part_c[tid] - sc;  // exclusive prefix of this chunk
  for (int i = lo; i < hi; ++i) {
    run_r += row_ptr[i + 1];
    run_c += col_ptr[i + 1];
    row_ptr[i + 1] = run_r;
    col_ptr[i + 1] = run_c;
  }
  if (tid == 0) { row_ptr[0] = 0; col_ptr[0] = 0; }
}

__global__ void __launch_bounds__(kMaskWarps * 32)
    blockmask_fill_kernel(const uint8_t* __restrict__ mask, int nT, const int32_t* __restrict__ row_ptr,
                          int32_t* __restrict__ col_idx, const int32_t* __restrict__ col_ptr,
                          int32_t* __restrict__ row_idx, long long head_stride) {
  mask += (size_t)blockIdx.y * nT * nT;
  row_ptr += blockIdx.y * head_stride;
  col_idx += blockIdx.y * head_stride;
  col_ptr += blockIdx.y * head_stride;
  row_idx += blockIdx.y * head_stride;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int rb = mask_row_blocks(nT);
  if ((int)blockIdx.x < rb) {
    const int i = blockIdx.x * kMaskWarps + warp;
    if (i >= nT) return;
    const uint8_t* r = mask + (size_t)i * nT;
    int pos = row_ptr[i];
    for (int x0 = 0; x0 < nT; x0 += 32) {
      const bool kept = x0 + lane < nT && r[x0 + lane] != 0;
      const unsigned bal = __ballot_sync(0xffffffffu, kept);
      const long long e = pos + __popc(bal & ((1u << lane) - 1u));  // a list holds at most nT * nT entries
      if (kept && in_bounds(e < (long long)nT * nT, kSiteMaskList)) col_idx[e] = x0 + lane;
      pos += __popc(bal);
    }
  } else {
    const int j = ((blockIdx.x - rb) * kMaskWarps + warp) * 32 + lane;
    if (j >= nT) return;
    int pos = col_ptr[j];
#pragma unroll 8
    for (int x = 0; x < nT; ++x)
      if (mask[(size_t)x * nT + j]) {
        if (in_bounds(pos < (long long)nT * nT, kSiteMaskList)) row_idx[pos] = x;
        ++pos;
      }
  }
}

// Debug-check self-test: one thread stores to indices 0..4 of a 4-entry array through in_bounds.  In an FA_DEBUG
// build the last index fails its check, which records kDevBounds and kSiteSelftest and skips that store; no access
// outside the array is made in either build.
__device__ int g_selftest_bounds_buf[4];
__global__ void selftest_bounds_kernel() {
  for (int i = 0; i <= 4; ++i)
    if (in_bounds(i < 4, kSiteSelftest)) g_selftest_bounds_buf[i & 3] = i;
}

// Waits on an mbarrier that nothing arrives on; the bounded wait must give up, record FA_ERR_TIMEOUT and return.
__global__ void selftest_wait_kernel(uint64_t budget_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_addr(&bar), 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  __syncthreads();
  wait_or_abort(ptx::smem_addr(&bar), 0, budget_ns, &abort_flag);
}

// Evaluates the FMA-pipe exp2 (ptx::exp2_fma) and the hardware ex2.approx on the same inputs, for accuracy tests.
__global__ void selftest_exp2_kernel(const float* __restrict__ x, float* __restrict__ out_fma,
                                     float* __restrict__ out_mufu, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    out_fma[i] = ptx::exp2_fma(x[i]);
    out_mufu[i] = ptx::ex2(x[i]);
  }
}

}  // namespace fa
