// fa_common.cuh -- pieces shared by the forward and backward kernels: the device status word, tile geometry,
// and the per-tile visibility rules (causal, key lengths, block-mask lists) applied at tile granularity.
#pragma once
#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include "ptx.cuh"

namespace fa {

constexpr int kTile = 128;  // rows of a Q tile and keys of a K/V tile

enum DeviceError : int { kDevOk = 0, kDevTimeout = 4, kDevBounds = 6 };

// One status word per device; the first error wins.  Read and cleared by fa_last_device_status().
__device__ int g_device_status = 0;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_status, 0, code); }

// ------------------------------------------------------------------------------------------------ debug checks
// FA_DEBUG builds (libfa_debug.so) check every index the kernels compute for a global-memory access against the
// extent of the buffer it addresses.  A failed check records kDevBounds in the status word and the site code
// below in g_bounds_site (first failure wins), and the caller skips the access, so the kernel neither faults nor
// traps.  Release builds compile the checks away (in_bounds is constant true).
#ifndef FA_DEBUG
#define FA_DEBUG 0
#endif
enum BoundsSite : int {
  kSiteFwdO = 1,         // forward O row store
  kSiteFwdLse = 2,       // forward LSE store
  kSiteSplitPart = 3,    // split-K/V partial O / LSE store
  kSiteCombine = 4,      // split-K/V combine O / LSE store
  kSiteFwd256 = 5,       // d = 256 forward O / LSE store
  kSiteBwdSide = 11,     // backward per-row fold / side data load
  kSiteBwdDq = 12,       // backward dQ partial-sum reduce box
  kSiteBwdKV = 13,       // backward dK / dV row store
  kSiteBwdPre = 14,      // backward preprocess row
  kSiteBwdDqConv = 15,   // dQ conversion row
  kSiteMaskList = 21,    // block-mask list entry
  kSiteSelftest = 99,    // fa_selftest_bounds
};
__device__ int g_bounds_site = 0;

__device__ __forceinline__ bool in_bounds(bool ok, int site) {
#if FA_DEBUG
  if (!ok) {
    record_error(kDevBounds);
    atomicCAS(&g_bounds_site, 0, site);
  }
  return ok;
#else
  (void)ok;
  (void)site;
  return true;
#endif
}

#ifndef FA_WAIT_HINT_NS
#define FA_WAIT_HINT_NS 0
#endif
// Bounded wait used by every pipeline role.  Gives up when the CTA's abort flag is raised by another role, or
// after `budget_ns` (then it records FA_ERR_TIMEOUT in the status word and raises the abort flag itself).
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, uint64_t budget_ns,
                                              volatile int* abort_flag) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  while (true) {
#if FA_WAIT_HINT_NS
    if (ptx::mbar_try_wait_sleep(bar, parity, FA_WAIT_HINT_NS)) return true;
#else
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
#endif
    if (*abort_flag) return false;
    if (ptx::globaltimer_ns() - t0 > budget_ns) {
      record_error(kDevTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}

// Number of keys visible to sequence b at all (key length clamped to N).
__device__ __forceinline__ int key_limit(const int32_t* key_lens, int b, int N) {
  if (key_lens == nullptr) return N;
  int l = key_lens[b];
  return l < 0 ? 0 : (l > N ? N : l);
}

// Exclusive end of the K/V tiles query tile i may see: tiles at or beyond it are fully hidden by the key
// limit or (causal) lie entirely above the diagonal.
__device__ __forceinline__ int kv_tile_end(int i, int kv_lim, bool causal) {
  int end = (kv_lim + kTile - 1) / kTile;
  if (causal && end > i + 1) end = i + 1;
  return end;
}

// The same when query row r sees keys c <= r + off (off = len_k - N_q aligns the queries with the end of the keys,
// as when a few new queries attend to a cache; off = 0 is kv_tile_end).
__device__ __forceinline__ int kv_tile_end_off(int i, int kv_lim, bool causal, int off) {
  int end = (kv_lim + kTile - 1) / kTile;
  if (causal) {
    const int last = i * kTile + kTile - 1 + off;  // last key the tile's last row may see
    const int e = last < 0 ? 0 : last / kTile + 1;
    if (end > e) end = e;
  }
  return end;
}

// Iterates, in ascending order, the K/V tiles visible to either of the two Q tiles a forward CTA owns.  Every
// role (loader, MMA issuer, softmax warps) walks the same sequence, so their pipelines stay in step.
//   dense : tile t sees [0, end_t)
//   sparse: tile t sees the ascending CSR list of its row, cut at end_t
struct PairTileIter {
  const int32_t* list[2];
  int len[2];   // dense: end_t; sparse: entries in list (already cut to < end_t)
  int pos[2];
  bool sparse;
  int next_dense;

  __device__ __forceinline__ void init_dense(int end0, int end1, int begin = 0) {
    sparse = false;
    len[0] = end0; len[1] = end1;
    pos[0] = pos[1] = 0;
    next_dense = begin;  // tiles [begin, end_t)
    list[0] = list[1] = nullptr;
  }

  __device__ __forceinline__ void init_sparse(const int32_t* row_ptr, const int32_t* col_idx, int row0, int nT,
                                              int end0, int end1) {
    sparse = true;
    next_dense = 0;
    for (int t = 0; t < 2; ++t) {
      const int r = row0 + t;
      pos[t] = 0;
      if (r >= nT) { list[t] = col_idx; len[t] = 0; continue; }
      const int a = row_ptr[r], b = row_ptr[r + 1];
      list[t] = col_idx + a;
      const int end = t == 0 ? end0 : end1;
      int n = 0;
      while (n < b - a && list[t][n] < end) ++n;  // lists are ascending
      len[t] = n;
    }
  }

  // Next visible tile j and a 2-bit mask of the Q tiles that see it.  Returns false when both are exhausted.
  __device__ __forceinline__ bool next(int& j, int& flags) {
    if (!sparse) {
      const int end = len[0] > len[1] ? len[0] : len[1];
      if (next_dense >= end) return false;
      j = next_dense++;
      flags = (j < len[0] ? 1 : 0) | (j < len[1] ? 2 : 0);
      return true;
    }
    const int a = pos[0] < len[0] ? list[0][pos[0]] : 0x7fffffff;
    const int b = pos[1] < len[1] ? list[1][pos[1]] : 0x7fffffff;
    if (a == 0x7fffffff && b == 0x7fffffff) return false;
    j = a < b ? a : b;
    flags = (a == j ? 1 : 0) | (b == j ? 2 : 0);
    if (a == j) ++pos[0];
    if (b == j) ++pos[1];
    return true;
  }

  // tiles tile t visits in a dense walk from 0 (sparse: its list length)
  __device__ __forceinline__ int count(int t) const { return len[t]; }
};

// Where the rows of one (b, h) live.  Dense [B, H, N, d]: rows 0..N-1 of plane b*H+h, keys limited by key_lens.
// Packed variable-length [total, H, d]: tokens cu[b] .. cu[b+1]-1 of head h, for queries and keys separately
// (the caller's cu_seqlens; values are clamped to [0, total] and lengths to the stated maximum, so a bad array
// cannot move an access out of range).  Positions r, c below are always relative to the sequence start.
struct SeqGeom {
  int q0, k0;  // first row (dense: 0) / token (packed) of the sequence
  int lq, lk;  // query rows, visible keys
};

__device__ __forceinline__ SeqGeom seq_geom(const int32_t* cu_q, const int32_t* cu_k, const int32_t* key_lens, int b,
                                            int N, int Nk, int total_q, int total_k) {
  SeqGeom g;
  if (cu_q != nullptr) {
    const int a = min(max(cu_q[b], 0), total_q), e = min(max(cu_q[b + 1], a), total_q);
    const int ak = min(max(cu_k[b], 0), total_k), ek = min(max(cu_k[b + 1], ak), total_k);
    g.q0 = a;
    g.lq = min(e - a, N);
    g.k0 = ak;
    g.lk = min(ek - ak, Nk);
  } else {
    g.q0 = 0;
    g.k0 = 0;
    g.lq = N;
    g.lk = key_limit(key_lens, b, N);
  }
  return g;
}

// One 128-row x 64-column box of a 16-bit tensor into shared memory.  Dense maps are {d, N, B*H} (row, plane);
// packed maps are {d, H, total} with a {64, 1, 128} box (head, token): both land as 128 rows of 128 bytes.
__device__ __forceinline__ void tma_rows(uint32_t dst, const CUtensorMap* map, int c, int row, int base, int bh, int h,
                                         bool packed, uint32_t bar) {
  if (packed)
    ptx::tma_load_3d(dst, map, 64 * c, h, base + row, bar);
  else
    ptx::tma_load_3d(dst, map, 64 * c, row, bh, bar);
}

// Persistent kernels: CTA c of G takes, in round r, unit r*G + c (r even) or r*G + G-1-c (r odd).  With units
// ordered longest first, this zigzag evens out the per-CTA work about as well as a greedy longest-first queue,
// without a global counter.
struct UnitSeq {
  int c, G, total, r;
  __device__ __forceinline__ void init(int total_units) {
    c = blockIdx.x;
    G = gridDim.x;
    total = total_units;
    r = 0;
  }
  __device__ __forceinline__ bool next(int& L) {
    while (r * G < total) {
      L = r * G + ((r & 1) ? G - 1 - c : c);
      ++r;
      if (L < total) return true;  // the last round may be partial
    }
    return false;
  }
};

// Number of SMs of the current device (cached per device).
inline cudaError_t device_sm_count(int dev, int* sms) {
  static std::atomic<int> cache[64];
  int v = cache[dev & 63].load();
  if (v == 0) {
    const cudaError_t e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    cache[dev & 63].store(v);
  }
  *sms = v;
  return cudaSuccess;
}

}  // namespace fa
