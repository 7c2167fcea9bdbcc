// fa_mask.cuh -- block-mask tile lists on the device (explainer page, block-sparse section: kept tiles are the
// only ones loaded), and the wait-timeout self-test kernel.
#pragma once
#include "fa_common.cuh"

namespace fa {

constexpr int kMaskThreads = 1024;
constexpr int kMaxMaskTiles = 8192;

// One CTA of 1024 threads.  Phase 1 counts kept tiles per row and per column, phase 2 turns the counts into
// exclusive prefix sums (row_ptr, col_ptr), phase 3 writes each row's columns and each column's rows in
// ascending order.  Integer only; the result is unique, so it must equal any correct CPU construction exactly.
// Per-head masks: CTA h reads mask + h*nT*nT and writes lists `head_stride` int32 further on (grid = number of
// masks; one mask shared by all heads: grid 1, stride 0).
__global__ void __launch_bounds__(kMaskThreads, 1)
    blockmask_lists_kernel(const uint8_t* __restrict__ mask, int nT, int32_t* __restrict__ row_ptr,
                           int32_t* __restrict__ col_idx, int32_t* __restrict__ col_ptr,
                           int32_t* __restrict__ row_idx, long long head_stride) {
  mask += (size_t)blockIdx.x * nT * nT;
  row_ptr += blockIdx.x * head_stride;
  col_idx += blockIdx.x * head_stride;
  col_ptr += blockIdx.x * head_stride;
  row_idx += blockIdx.x * head_stride;
  __shared__ int32_t part_r[kMaskThreads], part_c[kMaskThreads];
  const int tid = threadIdx.x;
  for (int i = tid; i < nT; i += kMaskThreads) {
    int cr = 0, cc = 0;
    for (int x = 0; x < nT; ++x) {
      cr += mask[(size_t)i * nT + x] != 0;  // row i
      cc += mask[(size_t)x * nT + i] != 0;  // column i (coalesced across threads)
    }
    row_ptr[i + 1] = cr;
    col_ptr[i + 1] = cc;
  }
  __syncthreads();
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
    const int cr = row_ptr[i + 1], cc = col_ptr[i + 1];
    run_r += cr;
    run_c += cc;
    row_ptr[i + 1] = run_r;
    col_ptr[i + 1] = run_c;
  }
  if (tid == 0) { row_ptr[0] = 0; col_ptr[0] = 0; }
  __syncthreads();
  for (int i = tid; i < nT; i += kMaskThreads) {
    int pr = row_ptr[i], pc = col_ptr[i];
    for (int x = 0; x < nT; ++x) {
      if (mask[(size_t)i * nT + x]) col_idx[pr++] = x;
      if (mask[(size_t)x * nT + i]) row_idx[pc++] = x;
    }
  }
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
