// fa_bwd.cuh -- backward kernels: gradients by recomputation from the saved logsumexp (sm_100a).
//
// Method (FlashAttention review page, claim C7 / E-recompute: the forward keeps only the softmax normalisation and
// the backward recomputes attention tiles on chip instead of reading an N x N matrix).  The pages print no backward
// equations; the reading used is the calculus of softmax attention for the loss sum(O * dO):
//     P = exp(scale * Q K^T - LSE),  D = rowsum(dO * O),  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - D),
//     dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three launches:
//   bwd_pre_kernel   D_r = sum_j dO_rj O_rj (fp32) for every row of a 128-padded row space; stores, per row, the
//                    fold rows of -LSE_r / scale and -D_r (three 16-bit parts each, see Fold) that the tensor core
//                    adds to S^T and dP^T (padded rows and rows with no visible key get the masked row, so their
//                    recomputed P is exactly 0); zeroes the fp32 dQ accumulator.  HBM-bound.
//   bwd_kernel       persistent, at most one CTA per SM; each CTA walks a share of the units (128-key tile j of
//                    one (b, h)) and, per unit, loops over the visible 128-row Q tiles i.
//                    Five tcgen05 GEMMs per (i, j): S^T = K Q^T and dP^T = V dO^T (recompute), dV += P^T dO (P^T read
//                    from TMEM), dK += dS^T Q and dQ_i = dS K (dS^T staged in shared memory, used K-major for dK and
//                    M-major for dQ).  dK, dV accumulate in TMEM for the whole loop.  Each dQ_i partial leaves
//                    through a 128-byte-swizzled shared-memory staging box and TMA bulk tensor reductions (add) into
//                    the fp32 accumulator: whole-line reductions in L2, no per-thread atomics.
//   bwd_dq_kernel    fp32 dQ accumulator -> 16-bit dQ.  HBM-bound.
//
// Roles in bwd_kernel (512 threads): warps 0-7 recompute P^T and dS^T (thread = key row = TMEM lane; warpgroup g
// takes queries [64g, 64g+64), so every SM sub-partition interleaves two such warps), warps 8-11 drain dQ_i
// (thread = query row) and write each unit's dK, dV, warp 12 issues MMAs, warp 13 issues TMA loads, warps 14-15
// only pad the fourth warpgroup.  At d = 64 the K/V tiles are double-buffered, so the next unit's load overlaps
// the current unit's last tiles; the epilogue overlaps the next unit's first scores.
// MMA order per Q tile i, so that the P^T warps recompute P_{i+1} while the tensor core finishes tile i:
//   d = 64:  [P^T_i] S^T_{i+1}, dV_i  [dS^T_i] dP^T_{i+1}, dK_i, dQ_i
//   d = 128: dP^T_i [P^T_i] dV_i, S^T_{i+1} [dS^T_i] dQ_i, dK_i      ([X] = wait until X is published)
// TMEM (512 columns): S^T [0,128); dP^T [128,256); dV [256,256+d); dK [256+d,256+2d).  d = 64: dQ_i [384,448) and
// P^T (16-bit pairs) [448,512).  d = 128 (no room left): P^T over S^T columns [0,32) and [64,96), dQ_i in the
// dP^T columns once read.
#pragma once
#include "fa_common.cuh"

namespace fa {

// Every kBwdExpFmaEvery-th pair of recomputed probabilities is exponentiated on the FMA pipe (ptx::exp2_fma);
// 0 = never.  Measured on B200: 1 pair in 8 or in 4 gains nothing in the backward, so it is off.
#ifndef FA_BWD_EXP_FMA_EVERY
#define FA_BWD_EXP_FMA_EVERY 0
#endif
constexpr int kBwdExpFmaEvery = FA_BWD_EXP_FMA_EVERY;
// Per-warpgroup register budgets (setmaxnreg): the two recompute warpgroups take FA_BWD_REGS_HIGH registers a
// thread, the drain warpgroup keeps 128 and the MMA / TMA warpgroup gives up the difference.  Measured on B200: at
// 136 / 112 the d = 64 kernel uses no local memory (128 for all: a stack frame and spills in the recompute loop) and
// the GPT-2 shape backward kernel goes from 388 to 403 TFLOP/s; 144 / 96 spills in the MMA / TMA warps.
#ifndef FA_BWD_SETMAXNREG
#define FA_BWD_SETMAXNREG 1
#endif
#ifndef FA_BWD_REGS_HIGH
#define FA_BWD_REGS_HIGH 136
#endif

template <int D>
struct BwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int kTileBytes = kTile * D * 2;       // 128 x D 16-bit tile
  static constexpr int kAugBytes = kTile * 16;           // 128 rows x 8 16-bit values: the tile's fold operand
  static constexpr int kSlotBytes = kTileBytes + kAugBytes;  // Q tile + its LSE fold rows, or dO tile + its D rows
  static constexpr int kSubTiles = D / 64;
  // Two rings of tile slots: Q tiles in kQSlots, dO tiles in kDoSlots (slots [kQSlots, kNumSlots)).  A dO slot is
  // freed by dV_i, early in tile i, so with d = 128 even one dO slot loads dO_{i+1} while S^T_{i+1}, dQ_i and dK_i
  // run; the Q slots are freed by the last MMA of their tile (dK_i), so they need the second slot.
  static constexpr int kQSlots = D == 128 ? 2 : 3;
  static constexpr int kDoSlots = D == 128 ? 1 : 3;
  static constexpr int kNumSlots = kQSlots + kDoSlots;
  static constexpr int kDsBytes = kTile * kTile * 2;      // dS^T, 128 keys x 128 queries
  static constexpr int kStageBytes = 4 * 4096;             // dQ staging: one 32 x 32 fp32 box per drain warp
  static constexpr int kKvBufs = D == 64 ? 2 : 1;           // K/V tile buffers: d = 64 prefetches the next unit's
  static constexpr int kOnesBytes = 2048;  // the fold's constant A operand (one core-matrix pair used, rest zero)
  static constexpr int kSmemBytes =
      kKvBufs * 2 * kTileBytes + kDsBytes + kNumSlots * kSlotBytes + kStageBytes + kOnesBytes + 1024;
  static constexpr int kThreads = 512;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  static constexpr bool kDqOwnCols = (D == 64);            // d = 64: dQ has its own columns
  static constexpr uint32_t kColDQ = kDqOwnCols ? 384 : kColDP;
  // P^T (16-bit pairs, 64 columns): its own columns [448, 512) for d = 64, so the next S^T may overwrite the S^T
  // columns as soon as they are read; for d = 128 inside the S^T columns ([0,32) and [64,96)).
  static constexpr uint32_t kColPT = kDqOwnCols ? 448 : kColS;
  static constexpr uint32_t kPtHalf = kDqOwnCols ? 32 : 64;  // column distance between the two query halves
};

// Per-row side data of the backward, in bytes: d <= 128 keeps, per padded row, the two fold rows of 8 16-bit
// values each (-LSE/scale and -D, split in three; see bwd_pre_kernel); d = 256 keeps -LSE2 and -scale * D as fp32.
inline size_t bwd_row_side_bytes(int d) { return d <= 128 ? 16 : 4; }
// Workspace layout: dq_acc [BH][Npad][d] fp32 | LSE side [BH][Npad] | D side [BH][Npad], each 256-B aligned
inline size_t bwd_workspace_bytes(int BH, int nT, int d) {
  const size_t npad = (size_t)nT * kTile;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  return al((size_t)BH * npad * d * 4) + 2 * al((size_t)BH * npad * bwd_row_side_bytes(d));
}

struct BwdArgs {
  void* dk;
  void* dv;
  float* dq_acc;
  const float* lse2;  // d = 256: -LSE2 per padded row;  d <= 128: the LSE fold rows (16 bytes per padded row)
  const float* Dv;    // d = 256: -scale * D per padded row;  d <= 128: the D fold rows
  const int32_t* key_lens;
  const int32_t* col_ptr;  // CSC of the block mask (nullptr: dense)
  const int32_t* row_idx;
  long long list_head_stride;  // per-head masks: int32 distance between heads' lists (0: one mask for all heads)
  const int32_t* cu_q;  // packed variable-length batch: cumulative sequence lengths (nullptr: dense [B,H,N,d])
  const int32_t* cu_k;
  int total_q, total_k;  // packed: token counts; dK, dV are [total_k, H, d]
  int H, N, nT, BH;  // nT = Q tiles of the padded row space (packed: of the longest query sequence)
  int Nk, nTk;       // key rows and K/V tiles per head (packed: of the longest key sequence)
  int dl;            // head dim of the tensors (32 / 96 run on the 64 / 128 kernels; dq_acc rows are dl wide)
  int causal;
  float scale;       // softmax scale
  float scale_log2;  // softmax scale * log2(e)
  uint64_t budget_ns;
};

// Ascending Q tiles visible to K/V tile j: [i0, nT), or the CSC list of column j cut to i >= i0.
struct ColTileIter {
  const int32_t* list;
  int len, pos, i0, dense_next;
  bool sparse;
  __device__ __forceinline__ void init(const int32_t* col_ptr, const int32_t* row_idx, int j, int nT, int first,
                                       bool visible) {
    pos = 0;
    i0 = first;
    dense_next = first;
    sparse = col_ptr != nullptr;
    list = nullptr;
    len = 0;
    if (!visible) {
      sparse = true;  // empty
      return;
    }
    if (sparse) {
      const int a = col_ptr[j], b = col_ptr[j + 1];
      list = row_idx + a;
      len = b - a;
      while (pos < len && list[pos] < first) ++pos;  // ascending
    } else {
      len = nT;
    }
  }
  __device__ __forceinline__ bool next(int& i) {
    if (sparse) {
      if (pos >= len) return false;
      i = list[pos++];
      return true;
    }
    if (dense_next >= len) return false;
    i = dense_next++;
    return true;
  }
  __device__ __forceinline__ int count() const { return sparse ? len - pos : len - dense_next; }
};

// ------------------------------------------------------------------------------------------------ preprocess
// Row r of a head needs D/8 lanes (16-byte loads of 8 16-bit values), so a warp covers 32*8/D rows per pass; the
// lanes of a row reduce with xor-shuffles inside their group.  Every padded row's dQ accumulator is zeroed with
// 16-byte stores.  Grid-stride over all padded rows of all heads.  Packed variable-length batches (cu_q non-null):
// O, dO are [total_q, H, d] and LSE [H, total_q]; the padded row space stays per (b, h), rows past the sequence's
// length get -LSE2 = -inf like padding.
// The fold (d <= 128).  The per-query terms of the recompute, -LSE_r / scale in the scores and -D_r in dP, are added
// by the tensor core: one more K = 16 step of S^T = K Q^T (and of dP^T = V dO^T) whose A operand holds the constant
// kFoldScale in columns 0-2 of every key row and whose B operand holds, for query r, the value w_r = x_r /
// kFoldScale split into three 16-bit parts (w = hi + mid + lo to about 24 bits) in columns 0-2.  The accumulator
// then holds S + x_r (fp32), so the P^T / dS^T warps need no per-query operand at all.  kFoldScale = 1 for bf16;
// 256 for fp16, whose 16-bit range would otherwise end at |x| = 65504 (beyond 256 * 65504 the fp16 fold saturates).
// Rows with no visible key (padding, fully masked rows) get w = -kFoldMasked: their P is exp2 of a huge negative
// number, exactly 0.
template <bool kBF16>
struct Fold {
  static constexpr float kScale = kBF16 ? 1.f : 256.f;
  static constexpr float kMasked = kBF16 ? 0x1p100f : 65504.f;
  static constexpr float kMax = kBF16 ? 3.0e38f : 65504.f;
  // 16 bytes: {hi, mid, lo, 0, 0, 0, 0, 0} of x / kScale
  static __device__ __forceinline__ uint4 row(float x) {
    const float w = fminf(fmaxf(x * (1.f / kScale), -kMax), kMax);
    const float hi = ptx::unpack2<kBF16>(ptx::pack2<kBF16>(w, 0.f)).x;
    const float r1 = w - hi;  // exact: hi is w rounded to fewer significand bits
    const float mid = ptx::unpack2<kBF16>(ptx::pack2<kBF16>(r1, 0.f)).x;
    return make_uint4(ptx::pack2<kBF16>(hi, mid), ptx::pack2<kBF16>(r1 - mid, 0.f), 0u, 0u);
  }
  static __device__ __forceinline__ uint4 masked_row() {
    return make_uint4(ptx::pack2<kBF16>(-kMasked, 0.f), 0u, 0u, 0u);
  }
};

template <int D, bool kBF16>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const void* __restrict__ o, const void* __restrict__ dout,
                                                      const float* __restrict__ lse, float* __restrict__ dq_acc,
                                                      float* __restrict__ lse2, float* __restrict__ Dv, int N,
                                                      int Npad, long long rows, float scale,
                                                      const int32_t* __restrict__ cu_q, int total_q, int H, int dl) {
  constexpr int kLanesPerRow = D / 8;          // 8 or 16
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;  // 4 or 2
  const int lane = threadIdx.x % 32;
  const int sub = lane / kLanesPerRow, l = lane % kLanesPerRow;
  const long long warp_global = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) / 32;
  for (long long row0 = warp_global * kRowsPerWarp; row0 < rows; row0 += nwarps * kRowsPerWarp) {
    const long long row = row0 + sub;
    const bool in = row < rows;
    const long long bh = in ? row / Npad : 0;
    const int r = in ? (int)(row % Npad) : 0;
    const SeqGeom g = seq_geom(cu_q, cu_q, nullptr, (int)(bh / H), N, N, total_q, total_q);
    const bool valid = r < g.lq;
    const size_t prow = cu_q ? (size_t)(g.q0 + r) * H + (size_t)(bh % H) : (size_t)bh * N + r;  // row of O, dO
    float dsum = 0.f;
    const bool col_ok = l * 8 < dl;  // lanes past the head dim (32 / 96 on the 64 / 128 kernels) hold nothing
    const size_t o_rows = cu_q ? (size_t)total_q * H : (size_t)(rows / Npad) * N;  // rows of O, dO (entries of LSE)
    (void)o_rows;
    if (in && valid && col_ok && in_bounds(prow < o_rows, kSiteBwdPre)) {
      const size_t off = prow * dl + (size_t)l * 8;
      const uint4 a = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(o) + off);
      const uint4 c = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(dout) + off);
      const uint32_t va[4] = {a.x, a.y, a.z, a.w}, vc[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const ptx::f32x2 x = ptx::unpack2<kBF16>(va[u]), y = ptx::unpack2<kBF16>(vc[u]);
        dsum = fmaf(x.x, y.x, dsum);
        dsum = fmaf(x.y, y.y, dsum);
      }
    }
#pragma unroll
    for (int m = kLanesPerRow / 2; m > 0; m >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, m);
    if (in) {
      if (col_ok) {
        float4* acc = reinterpret_cast<float4*>(dq_acc + row * dl);
        acc[2 * l] = make_float4(0.f, 0.f, 0.f, 0.f);
        acc[2 * l + 1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (l == 0) {
        const size_t li = cu_q ? (size_t)(bh % H) * total_q + g.q0 + r : (size_t)bh * N + r;
        const float lv = valid && in_bounds(li < o_rows, kSiteBwdPre) ? lse[li] : -INFINITY;
        if constexpr (D <= 128) {
          // the fold rows: -LSE / scale and -D (padded row or no visible key: the masked row, P = 0)
          reinterpret_cast<uint4*>(lse2)[row] = lv != -INFINITY ? Fold<kBF16>::row(-lv / scale) : Fold<kBF16>::masked_row();
          reinterpret_cast<uint4*>(Dv)[row] = Fold<kBF16>::row(-dsum);
        } else {
          // padded row or no visible key: recomputed P = exp2(x - inf) = 0
          lse2[row] = lv != -INFINITY ? -lv * 1.4426950408889634f : -INFINITY;
          Dv[row] = -scale * dsum;
        }
      }
    }
  }
}

// ------------------------------------------------------------------------------------------------ dQ convert
// Each thread converts 8 consecutive elements (two 16-byte loads, one 16-byte store).  Dense: over the N-row
// output.  Packed variable-length: over the padded rows, writing those inside their sequence to [total_q, H, d].
template <int D, bool kBF16>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ dq_acc, void* __restrict__ dq, int N,
                                                     int Npad, long long total_vec8, const int32_t* __restrict__ cu_q,
                                                     int total_q, int H, int dl) {
  for (long long v = (long long)blockIdx.x * blockDim.x + threadIdx.x; v < total_vec8;
       v += (long long)gridDim.x * blockDim.x) {
    const long long e = v * 8;
    const long long row = e / dl;  // dense: bh * N + r; packed: bh * Npad + r
    const int c = (int)(e % dl);
    const long long bh = row / (cu_q ? Npad : N);
    const int r = (int)(row % (cu_q ? Npad : N));
    size_t out_e = (size_t)e;
    if (cu_q) {
      const SeqGeom g = seq_geom(cu_q, cu_q, nullptr, (int)(bh / H), N, N, total_q, total_q);
      if (r >= g.lq) continue;
      out_e = ((size_t)(g.q0 + r) * H + (size_t)(bh % H)) * dl + c;
    }
    // extents checked in FA_DEBUG builds: rows of the fp32 accumulator ([BH][Npad]) and elements of dQ
    const long long rows_v = total_vec8 * 8 / dl;  // dense: BH * N; packed: BH * Npad
    const size_t acc_rows = cu_q ? (size_t)rows_v : (size_t)(rows_v / N) * Npad;
    const size_t out_elems = cu_q ? (size_t)total_q * H * dl : (size_t)total_vec8 * 8;
    if (!in_bounds((size_t)bh * Npad + r < acc_rows && out_e + 8 <= out_elems, kSiteBwdDqConv)) continue;
    (void)acc_rows;
    (void)out_elems;
    const float4* src = reinterpret_cast<const float4*>(dq_acc + ((size_t)bh * Npad + r) * dl + c);
    const float4 a = src[0], b = src[1];
    uint4 out;
    out.x = ptx::pack2<kBF16>(a.x, a.y);
    out.y = ptx::pack2<kBF16>(a.z, a.w);
    out.z = ptx::pack2<kBF16>(b.x, b.y);
    out.w = ptx::pack2<kBF16>(b.z, b.w);
    *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(dq) + out_e) = out;
  }
}

// ------------------------------------------------------------------------------------------------ main kernel
// Units of work are (K/V tile j, head bh), ordered j-major so that the longest causal columns come first; the
// kernel is persistent and walks them with UnitSeq.
struct BwdUnit {
  int j, bh, h, kv_lim, nTq;
  SeqGeom g;
  bool visible;  // some key of the tile is visible to someone
};

__device__ __forceinline__ BwdUnit bwd_unit(int L, const BwdArgs& a) {
  BwdUnit u;
  u.j = L / a.BH;
  u.bh = L % a.BH;
  u.h = u.bh % a.H;
  u.g = seq_geom(a.cu_q, a.cu_k, a.key_lens, u.bh / a.H, a.N, a.Nk, a.total_q, a.total_k);
  u.kv_lim = u.g.lk;
  u.nTq = (u.g.lq + kTile - 1) / kTile;
  u.visible = u.j * kTile < u.kv_lim && u.nTq > 0;
  return u;
}

template <int D, bool kBF16>
__global__ void __launch_bounds__(512, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
               const __grid_constant__ CUtensorMap map_dq, const BwdArgs args) {
  using C = BwdCfg<D>;
  constexpr int NS = C::kNumSlots, KB = C::kKvBufs;
  // ring position k = 2 t + v of the t-th Q tile processed (v = 0: its Q tile, v = 1: its dO tile)
  auto pos_slot = [](int k) { return (k & 1) ? C::kQSlots + (k >> 1) % C::kDoSlots : (k >> 1) % C::kQSlots; };
  auto pos_phase = [](int k) {
    return (uint32_t)(((k & 1) ? (k >> 1) / C::kDoSlots : (k >> 1) / C::kQSlots) & 1);
  };
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;                               // KB x (K tile, V tile)
  uint8_t* sDS = smem + KB * 2 * C::kTileBytes;
  uint8_t* sRing = sDS + C::kDsBytes;
  uint8_t* sStage = sRing + NS * C::kSlotBytes;  // 1024-aligned: slot bytes are multiples of 1024
  uint8_t* sOnes = sStage + C::kStageBytes;
  auto sK = [&](int kb) { return sKV + kb * 2 * C::kTileBytes; };
  auto sV = [&](int kb) { return sKV + kb * 2 * C::kTileBytes + C::kTileBytes; };

  __shared__ __align__(8) uint64_t bar_kv[KB], bar_kv_free[KB], bar_full[NS], bar_empty[NS], bar_s, bar_dp, bar_p,
      bar_ds, bar_dq_full, bar_dq_free, bar_ds_free, bar_pt_free, bar_dv_done, bar_done, bar_dv_free, bar_dk_free,
      bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  volatile int* abortp = &abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  // warps 0-7: P^T/dS^T (two warpgroups, one per 64-query half), 8-11: dQ drain and the dK/dV epilogue,
  // 12: MMA, 13: TMA, 14-15: idle
  constexpr int kWarpDrain = 8, kWarpMma = 12, kWarpLoad = 13;
  const bool causal = args.causal != 0;
  const int Npad = args.nT * kTile;
  const int total_units = args.nTk * args.BH;
  const bool packed = args.cu_q != nullptr;

  if (threadIdx.x == 0) {
    for (int k = 0; k < KB; ++k) {
      ptx::mbar_init(ptx::smem_addr(&bar_kv[k]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_kv_free[k]), 1);
    }
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(ptx::smem_addr(&bar_full[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_empty[s]), 1);
    }
    ptx::mbar_init(ptx::smem_addr(&bar_s), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dp), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_p), 256);
    ptx::mbar_init(ptx::smem_addr(&bar_ds), 256);
    ptx::mbar_init(ptx::smem_addr(&bar_dq_full), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dq_free), 128);
    ptx::mbar_init(ptx::smem_addr(&bar_ds_free), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_pt_free), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dv_done), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_done), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dv_free), 128);
    ptx::mbar_init(ptx::smem_addr(&bar_dk_free), 128);
    ptx::mbar_init(ptx::smem_addr(&bar_drain), 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_addr(&tmem_base_sh), C::kTmemCols);
    ptx::tmem_relinquish();
  }
  // The fold's A operand: kScale in columns 0-2 of the 8 rows of one core matrix (bytes [0,128)), zeros in its
  // second K chunk (bytes [128,256)); every 8-row group of the 128 key rows reads that same pair (group stride 0).
  if (threadIdx.x < C::kOnesBytes / 16) {
    const uint32_t f2 = ptx::pack2<kBF16>(Fold<kBF16>::kScale, Fold<kBF16>::kScale);
    const uint32_t f1 = ptx::pack2<kBF16>(Fold<kBF16>::kScale, 0.f);
    *reinterpret_cast<uint4*>(sOnes + threadIdx.x * 16) = threadIdx.x < 8 ? make_uint4(f2, f1, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // Register budgets per warpgroup when FA_BWD_SETMAXNREG is set (launched with 128 each): the recompute
  // warpgroups hold a tile row of scores, probabilities and gradients, the MMA / TMA warpgroup needs few
  // (kBwdRegsLow + 2 * kBwdRegsHigh + 128 = 4 x 128).  Each role changes its budget at the top of its own branch.
  constexpr int kBwdRegsHigh = FA_BWD_REGS_HIGH, kBwdRegsLow = 512 - 128 - 2 * FA_BWD_REGS_HIGH;
  static_assert(2 * kBwdRegsHigh + 128 + kBwdRegsLow <= 4 * 128, "register split exceeds the launch budget");

  // Every role walks the same unit sequence and, per unit, the same Q-tile list; counters that index barrier
  // phases and ring slots run on across units.  Units without a visible Q tile load and compute nothing (the
  // epilogue writes zero dK, dV for them).
  UnitSeq us;
  us.init(total_units);
  int L;

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------------------------------------ TMA producer
#if FA_BWD_SETMAXNREG
    ptx::setmaxnreg_dec<kBwdRegsLow>();
#endif
    if (lane == 0) {
      ptx::prefetch_tensormap(&map_q);
      ptx::prefetch_tensormap(&map_do);
      ptx::prefetch_tensormap(&map_k);
      ptx::prefetch_tensormap(&map_v);
      int n = 0, ku = 0;
      bool ok = true;
      while (ok && us.next(L)) {
        const BwdUnit u = bwd_unit(L, args);
        ColTileIter it;
        it.init(args.col_ptr ? args.col_ptr + u.h * args.list_head_stride : nullptr,
                args.row_idx + u.h * args.list_head_stride, u.j, u.nTq, causal ? u.j : 0, u.visible);
        if (it.count() == 0) continue;
        const int kb = ku % KB;
        // the buffer's previous K/V tiles must have been read by every MMA of their unit
        if (ku >= KB &&
            !wait_or_abort(ptx::smem_addr(&bar_kv_free[kb]), ((ku / KB) - 1) & 1, args.budget_ns, abortp)) {
          ok = false;
          break;
        }
        const uint32_t bkv = ptx::smem_addr(&bar_kv[kb]);
        ptx::mbar_arrive_expect_tx(bkv, 2 * C::kTileBytes);
        for (int c = 0; c < C::kSubTiles; ++c) {
          tma_rows(ptx::smem_addr(sK(kb) + c * 16384), &map_k, c, u.j * kTile, u.g.k0, u.bh, u.h, packed, bkv);
          tma_rows(ptx::smem_addr(sV(kb) + c * 16384), &map_v, c, u.j * kTile, u.g.k0, u.bh, u.h, packed, bkv);
        }
        int i;
        while (ok && it.next(i)) {
          for (int v = 0; v < 2; ++v) {  // v = 0: Q_i and its LSE fold rows, v = 1: dO_i and its D fold rows
            const int s = pos_slot(n);
            const uint32_t ph = pos_phase(n);
            if (!wait_or_abort(ptx::smem_addr(&bar_empty[s]), ph ^ 1, args.budget_ns, abortp)) { ok = false; break; }
            const uint32_t bf = ptx::smem_addr(&bar_full[s]);
            uint8_t* slot = sRing + s * C::kSlotBytes;
            const size_t row0 = (size_t)u.bh * Npad + (size_t)i * kTile;
            // the 128 fold rows lie inside the [BH][Npad] side arrays (a skipped load is left out of the byte count)
            const bool side_ok = in_bounds(row0 + kTile <= (size_t)args.BH * Npad, kSiteBwdSide);
            ptx::mbar_arrive_expect_tx(bf, C::kTileBytes + (side_ok ? C::kAugBytes : 0));
            for (int c = 0; c < C::kSubTiles; ++c)
              tma_rows(ptx::smem_addr(slot + c * 16384), v == 0 ? &map_q : &map_do, c, i * kTile, u.g.q0, u.bh, u.h,
                       packed, bf);
            const uint8_t* side = reinterpret_cast<const uint8_t*>(v == 0 ? args.lse2 : args.Dv) + row0 * 16;
            if (side_ok) ptx::bulk_load(ptx::smem_addr(slot + C::kTileBytes), side, C::kAugBytes, bf);
            ++n;
          }
        }
        ++ku;
      }
      // Let every copy this thread issued land before the CTA can exit (immediate in the normal path).
      for (int k = (ku > KB ? ku - KB : 0); k < ku; ++k)
        ptx::mbar_wait(ptx::smem_addr(&bar_kv[k % KB]), (k / KB) & 1, args.budget_ns);
      // (the last positions that used each slot: kQSlots Q tiles, kDoSlots dO tiles)
      for (int k = n - 2 * C::kQSlots; k < n; k += 2)
        if (k >= 0) ptx::mbar_wait(ptx::smem_addr(&bar_full[pos_slot(k)]), pos_phase(k), args.budget_ns);
      for (int k = n + 1 - 2 * C::kDoSlots; k < n; k += 2)
        if (k >= 0) ptx::mbar_wait(ptx::smem_addr(&bar_full[pos_slot(k)]), pos_phase(k), args.budget_ns);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------------------------------ MMA issuer
#if FA_BWD_SETMAXNREG
    ptx::setmaxnreg_dec<kBwdRegsLow>();
#endif
    if (lane == 0) {
      constexpr uint32_t id_sq = ptx::idesc_f16(kBF16, false, false, 128, 128);  // S^T, dP^T
      constexpr uint32_t id_dv = ptx::idesc_f16(kBF16, false, true, 128, D);     // dV (A from TMEM), dK
      constexpr uint32_t id_dq = ptx::idesc_f16(kBF16, true, true, 128, D);      // dQ
      // Operand descriptors are built once; each MMA advances one by a constant (K-major: +32 B per 16-element K
      // step inside a 64-element sub-tile, +16 KB per sub-tile; M/N-major: +2 KB per 16-row K step).
      const uint64_t dds_k = ptx::sw128_desc(ptx::smem_addr(sDS), 16, 1024);      // dS^T, K-major (dK)
      const uint64_t dds_mn = ptx::sw128_desc(ptx::smem_addr(sDS), 16384, 1024);  // dS, M-major (dQ)
      const uint64_t dring_k = ptx::sw128_desc(ptx::smem_addr(sRing), 16, 1024);
      const uint64_t dring_mn = ptx::sw128_desc(ptx::smem_addr(sRing), 16384, 1024);
      auto slot_off = [&](int k) { return (uint32_t)(pos_slot(k) * C::kSlotBytes); };
      auto slot_full = [&](int k) { return ptx::smem_addr(&bar_full[pos_slot(k)]); };
      auto slot_empty = [&](int k) { return ptx::smem_addr(&bar_empty[pos_slot(k)]); };
      auto slot_phase = [&](int k) { return pos_phase(k); };
      constexpr auto kstep = [](int kk) { return (uint32_t)((kk / 4) * 16384 + (kk % 4) * 32); };
      // the fold step: A = the constant tile (K chunks 128 B apart, 8-row groups all alike), B = the slot's fold
      // rows (16 bytes per query row, contiguous; the second K chunk repeats the first, where A holds zeros)
      const uint64_t d_ones = ptx::plain_desc(ptx::smem_addr(sOnes), 128, 0);
      const uint64_t d_fold = ptx::plain_desc(ptx::smem_addr(sRing + C::kTileBytes), 0, 128);
      uint64_t dk_k = 0, dk_mn = 0, dv_k = 0;  // K_j (K-major for S^T, M/N-major for dQ), V_j (K-major for dP^T)
      // S^T = K Q^T for the Q tile in ring position kq
      auto issue_s = [&](int kq) -> bool {
        if (!wait_or_abort(slot_full(kq), slot_phase(kq), args.budget_ns, abortp)) return false;
        ptx::tc_fence_after();
        const uint64_t dq = ptx::desc_advance(dring_k, slot_off(kq));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ptx::mma_ss(tmem + C::kColS, ptx::desc_advance(dk_k, kstep(kk)), ptx::desc_advance(dq, kstep(kk)), id_sq,
                      kk > 0 ? 1u : 0u);
        ptx::mma_ss(tmem + C::kColS, d_ones, ptx::desc_advance(d_fold, slot_off(kq)), id_sq, 1u);  // + (-LSE / scale)
        ptx::mma_commit(ptx::smem_addr(&bar_s));
        return true;
      };
      // dP^T = V dO_i^T for the dO tile in ring position ko
      auto issue_dp = [&](int ko) -> bool {
        if (!wait_or_abort(slot_full(ko), slot_phase(ko), args.budget_ns, abortp)) return false;
        ptx::tc_fence_after();
        const uint64_t ddo = ptx::desc_advance(dring_k, slot_off(ko));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ptx::mma_ss(tmem + C::kColDP, ptx::desc_advance(dv_k, kstep(kk)), ptx::desc_advance(ddo, kstep(kk)), id_sq,
                      kk > 0 ? 1u : 0u);
        ptx::mma_ss(tmem + C::kColDP, d_ones, ptx::desc_advance(d_fold, slot_off(ko)), id_sq, 1u);  // + (-D)
        ptx::mma_commit(ptx::smem_addr(&bar_dp));
        return true;
      };
      // dV += P^T dO_i   (P^T from TMEM, query half kk/4 at kColPT + kPtHalf*(kk/4); dO_i M/N-major)
      auto issue_dv = [&](int ko, bool first) {
        const uint64_t ddo = ptx::desc_advance(dring_mn, slot_off(ko));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          ptx::mma_ts(tmem + C::kColDV, tmem + C::kColPT + (kk / 4) * C::kPtHalf + (kk % 4) * 8,
                      ptx::desc_advance(ddo, kk * 2048), id_dv, (!first || kk > 0) ? 1u : 0u);
        ptx::mma_commit(slot_empty(ko));  // dO_i no longer needed
      };
      // dK += dS^T Q_i  (dS^T K-major in shared memory, Q_i M/N-major)
      auto issue_dk = [&](int kq, bool first) {
        const uint64_t dq = ptx::desc_advance(dring_mn, slot_off(kq));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          ptx::mma_ss(tmem + C::kColDK, ptx::desc_advance(dds_k, kstep(kk)), ptx::desc_advance(dq, kk * 2048), id_dv,
                      (!first || kk > 0) ? 1u : 0u);
        ptx::mma_commit(slot_empty(kq));  // Q_i (and its fold rows) no longer needed
      };
      // dQ_i = dS K_j  (dS read M-major from the dS^T tile)
      auto issue_dq = [&]() {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          ptx::mma_ss(tmem + C::kColDQ, ptx::desc_advance(dds_mn, kk * 2048), ptx::desc_advance(dk_mn, kk * 2048),
                      id_dq, kk > 0 ? 1u : 0u);
        ptx::mma_commit(ptx::smem_addr(&bar_dq_full));
      };
      int gi = 0, ku = 0;  // Q tiles and non-empty units processed so far
      bool ok = true;
      while (ok && us.next(L)) {
        const BwdUnit u = bwd_unit(L, args);
        ColTileIter it;
        it.init(args.col_ptr ? args.col_ptr + u.h * args.list_head_stride : nullptr,
                args.row_idx + u.h * args.list_head_stride, u.j, u.nTq, causal ? u.j : 0, u.visible);
        if (it.count() == 0) continue;
        const int kb = ku % KB;
        dk_k = ptx::sw128_desc(ptx::smem_addr(sK(kb)), 16, 1024);
        dk_mn = ptx::sw128_desc(ptx::smem_addr(sK(kb)), 16384, 1024);
        dv_k = ptx::sw128_desc(ptx::smem_addr(sV(kb)), 16, 1024);
        // dV and dK start over in TMEM: the epilogue must have read the previous unit's (dV and dK are released
        // separately: dV as soon as the previous unit's last dV MMA is done, so this unit's first dV rarely waits)
        auto acc_ready = [&](uint64_t& bar_free) -> bool {
          if (ku == 0) return true;
          if (!wait_or_abort(ptx::smem_addr(&bar_free), (ku - 1) & 1, args.budget_ns, abortp)) return false;
          ptx::tc_fence_after();
          return true;
        };
        if (!(ok = wait_or_abort(ptx::smem_addr(&bar_kv[kb]), (ku / KB) & 1, args.budget_ns, abortp))) break;
        ptx::tc_fence_after();
        int i, li = 0;
        bool have = it.next(i);
        if constexpr (C::kDqOwnCols) {
          // d = 64.  Per Q tile i:  [P^T_i published] S^T_{i+1}, dV_i  [dS^T_i published] dP^T_{i+1}, dK_i, dQ_i.
          // The next tile's S^T and dP^T are issued as soon as their TMEM columns have been read, so the P^T/dS^T
          // warps find them complete when they get there.
          if (!(ok = issue_s(2 * gi))) break;
          if (!(ok = issue_dp(2 * gi + 1))) break;
          while (ok && have) {
            const int kq = 2 * gi, ko = 2 * gi + 1;
            const uint32_t ph = gi & 1, ph_prev = (gi - 1) & 1;
            if (!(ok = wait_or_abort(ptx::smem_addr(&bar_p), ph, args.budget_ns, abortp))) break;
            ptx::tc_fence_after();
            int inext;
            const bool have_next = it.next(inext);
            if (have_next && !(ok = issue_s(kq + 2))) break;
            if (li == 0 && !(ok = acc_ready(bar_dv_free))) break;
            issue_dv(ko, li == 0);
            ptx::mma_commit(ptx::smem_addr(&bar_pt_free));
            if (!have_next) ptx::mma_commit(ptx::smem_addr(&bar_dv_done));  // this unit's dV is final
            if (!(ok = wait_or_abort(ptx::smem_addr(&bar_ds), ph, args.budget_ns, abortp))) break;
            ptx::tc_fence_after();
            if (have_next && !(ok = issue_dp(ko + 2))) break;
            if (li == 0 && !(ok = acc_ready(bar_dk_free))) break;
            issue_dk(kq, li == 0);
            if (gi > 0 && !(ok = wait_or_abort(ptx::smem_addr(&bar_dq_free), ph_prev, args.budget_ns, abortp)))
              break;
            ptx::tc_fence_after();
            issue_dq();
            ptx::mma_commit(ptx::smem_addr(&bar_ds_free));
            ++gi;
            ++li;
            have = have_next;
            i = inext;
          }
        } else {
          // d = 128.  Per Q tile i: dP^T_i, dV_i, S^T_{i+1}, dQ_i, dK_i.  dQ_i occupies the dP^T columns, so dP^T_i
          // waits until the drain warps have read dQ_{i-1}; dQ_i goes before dK_i to start that drain sooner.
          // S^T_{i+1} overwrites P^T_i only after dV_i (MMA order).
          if (!(ok = issue_s(2 * gi))) break;
          while (ok && have) {
            const int kq = 2 * gi, ko = 2 * gi + 1;
            const uint32_t ph = gi & 1, ph_prev = (gi - 1) & 1;
            if (gi > 0 && !(ok = wait_or_abort(ptx::smem_addr(&bar_dq_free), ph_prev, args.budget_ns, abortp)))
              break;
            ptx::tc_fence_after();
            if (!(ok = issue_dp(ko))) break;
            if (!(ok = wait_or_abort(ptx::smem_addr(&bar_p), ph, args.budget_ns, abortp))) break;
            ptx::tc_fence_after();
            if (li == 0 && !(ok = acc_ready(bar_dv_free))) break;
            issue_dv(ko, li == 0);
            int inext;
            const bool have_next = it.next(inext);
            if (!have_next) ptx::mma_commit(ptx::smem_addr(&bar_dv_done));  // this unit's dV is final
            if (have_next && !(ok = issue_s(kq + 2))) break;
            if (!(ok = wait_or_abort(ptx::smem_addr(&bar_ds), ph, args.budget_ns, abortp))) break;
            ptx::tc_fence_after();
            issue_dq();
            if (li == 0 && !(ok = acc_ready(bar_dk_free))) break;
            issue_dk(kq, li == 0);
            ptx::mma_commit(ptx::smem_addr(&bar_ds_free));
            ++gi;
            ++li;
            have = have_next;
            i = inext;
          }
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&bar_done));        // dK of this unit is final (and every MMA before it)
        ptx::mma_commit(ptx::smem_addr(&bar_kv_free[kb]));  // K_j, V_j no longer read
        ++ku;
      }
      ptx::mma_commit(ptx::smem_addr(&bar_drain));
      ptx::mbar_wait(ptx::smem_addr(&bar_drain), 0, args.budget_ns);
    }
  } else if (warp < kWarpDrain) {
    // ------------------------------------------------------------------------------------------ P^T / dS^T warps
    // Warpgroup g handles queries [64g, 64g+64) of every key row; the 4 warps of a group cover the 128 key rows.
#if FA_BWD_SETMAXNREG
    ptx::setmaxnreg_inc<kBwdRegsHigh>();
#endif
    const int g = warp / 4, quarter = warp % 4;
    const int c = quarter * 32 + lane;  // key row within the tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const ptx::f32x2 sl2v{args.scale_log2, args.scale_log2}, sc2{args.scale, args.scale};
    int gi = 0;
    bool ok = true;
    while (ok && us.next(L)) {
      const BwdUnit u = bwd_unit(L, args);
      ColTileIter it;
      it.init(args.col_ptr ? args.col_ptr + u.h * args.list_head_stride : nullptr,
                args.row_idx + u.h * args.list_head_stride, u.j, u.nTq, causal ? u.j : 0, u.visible);
      const int j = u.j, kv_lim = u.kv_lim;
      const int gc = j * kTile + c;  // key index in the sequence
      int i;
      while (it.next(i)) {
        const uint32_t ph = gi & 1;
        // S^T arrives with -LSE / scale already added per query column (the fold), dP^T with -D
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_s), ph, args.budget_ns, abortp));
        if (!ok) break;
        ptx::tc_fence_after();
        const bool masked = (causal && i == j) || (j + 1) * kTile > kv_lim;
        // visible queries of key gc: r >= gc (causal) and the key itself below the key limit
        const int rmin = causal ? gc - i * kTile - 64 * g : 0;  // first visible query column within this half
        const bool key_ok = gc < kv_lim;
        uint32_t pk[32];  // P^T of this half, 16-bit pairs
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t sr[32];
          ptx::tmem_ld32(tmem + lane_base + C::kColS + 64 * g + 32 * h, sr);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const int r0 = 32 * h + 2 * v;
            const bool emu = kBwdExpFmaEvery > 0 && v % (kBwdExpFmaEvery > 0 ? kBwdExpFmaEvery : 1) == 0;
            // (S - LSE / scale) * scale * log2(e) = log2 P
            const ptx::f32x2 x = ptx::mul2({__uint_as_float(sr[2 * v]), __uint_as_float(sr[2 * v + 1])}, sl2v);
            float p0 = emu ? ptx::exp2_fma(x.x) : ptx::ex2(x.x);
            float p1 = emu ? ptx::exp2_fma(x.y) : ptx::ex2(x.y);
            if (masked) {
              if (!key_ok || r0 < rmin) p0 = 0.f;
              if (!key_ok || r0 + 1 < rmin) p1 = 0.f;
            }
            pk[16 * h + v] = ptx::pack2<kBF16>(p0, p1);
          }
        }
        // P^T of this half (2 queries per 32-bit column) goes to kColPT + kPtHalf*g.  d = 128: inside the S^T
        // columns this warpgroup has just read, never over columns the other warpgroup may still be reading.
        // d = 64: its own columns, free once dV_{i-1} has read P^T_{i-1}.
        if (C::kDqOwnCols && gi > 0) {
          ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_pt_free), (gi - 1) & 1, args.budget_ns,
                                                      abortp));
          if (!ok) break;
          ptx::tc_fence_after();
        }
        ptx::tmem_st32(tmem + lane_base + C::kColPT + C::kPtHalf * g, pk);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&bar_p));
        // dS^T = P^T * (dP^T - D) * scale, written 16-bit into sub-tile g of the swizzled dS^T tile
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_dp), ph, args.budget_ns, abortp));
        if (ok && gi > 0)
          ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_ds_free), (gi - 1) & 1, args.budget_ns,
                                                      abortp));
        if (!ok) break;
        ptx::tc_fence_after();
        uint8_t* rowp = sDS + g * 16384 + c * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t dr[32];
          ptx::tmem_ld32(tmem + lane_base + C::kColDP + 64 * g + 32 * h, dr);
          ptx::tmem_ld_wait();
          uint32_t o[16];
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            // dS = P * (dP - D) * scale, P as the 16-bit values dV used (dP - D from the fold)
            const ptx::f32x2 t = ptx::mul2({__uint_as_float(dr[2 * v]), __uint_as_float(dr[2 * v + 1])}, sc2);
            const ptx::f32x2 ds = ptx::mul2(ptx::unpack2<kBF16>(pk[16 * h + v]), t);
            o[v] = ptx::pack2<kBF16>(ds.x, ds.y);
          }
          // queries 32h .. 32h+31 of this half: 16-byte chunks 4h .. 4h+3 of row c (128-byte swizzle)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int chunk = (4 * h + v) ^ (c & 7);
            *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          }
        }
        ptx::fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&bar_ds));
        ++gi;
      }
    }
  } else if (warp < kWarpMma) {
    // ------------------------------------------------------------------------------------------ drain warps
    // dQ_i: each warp owns 32 query rows (its TMEM lanes).  Per 32-column chunk it writes a 32 x 32 fp32 box into
    // its staging buffer in the 128-byte-swizzled layout of the dq_acc tensor map (16-byte chunk k of row r lands at
    // k ^ (r % 8): conflict-free), then one lane issues a TMA reduce-add of that box into dq_acc.  The TMEM region
    // is released as soon as the last columns are in registers.
    // dK, dV epilogue: each warp reads its 32 key rows of dV as soon as the unit's last dV MMA is done (before the
    // last dQ drain) and of dK after the unit's last MMA (dK already carries the softmax scale through dS), releases
    // each accumulator to the next unit as soon as it is read, and stores them 16-bit.
    const int wq = warp - kWarpDrain;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    uint8_t* stage = sStage + wq * 4096;
    const uint32_t stage_addr = ptx::smem_addr(stage);
    int gi = 0, ku = 0;
    bool ok = true;
    while (ok && us.next(L)) {
      const BwdUnit u = bwd_unit(L, args);
      ColTileIter it;
      it.init(args.col_ptr ? args.col_ptr + u.h * args.list_head_stride : nullptr,
                args.row_idx + u.h * args.list_head_stride, u.j, u.nTq, causal ? u.j : 0, u.visible);
      const int n_iters = it.count();
      const int gc = u.j * kTile + wq * 32 + lane;  // key row of this lane in the dK, dV epilogue
      // dense: every row of the head (keys past a key length get zero); packed: the sequence's own keys only
      const bool row_ok = packed ? gc < u.g.lk : gc < args.N;
      const size_t krow = packed ? (size_t)(u.g.k0 + gc) * args.H + u.h : (size_t)u.bh * args.N + gc;
      const size_t kv_rows = packed ? (size_t)args.total_k * args.H : (size_t)args.BH * args.N;  // rows of dK, dV
      (void)kv_rows;
      // dV (is_dk false) or dK of this unit: read out of TMEM chunk by chunk, release the columns to the next unit
      // after the last read, store 16-bit; a unit with no visible query writes zeros
      auto epilogue = [&](bool is_dk) {
        uint8_t* row = reinterpret_cast<uint8_t*>(is_dk ? args.dk : args.dv) + krow * args.dl * 2;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          if (n_iters > 0) {
            ptx::tmem_ld32(tmem + lane_base + (is_dk ? C::kColDK : C::kColDV) + cc * 32, r);
            ptx::tmem_ld_wait();
            if (cc == D / 32 - 1) {
              ptx::tc_fence_before();
              ptx::mbar_arrive(ptx::smem_addr(is_dk ? &bar_dk_free : &bar_dv_free));
            }
          } else {
#pragma unroll
            for (int v = 0; v < 32; ++v) r[v] = 0u;  // no visible query: zero gradient
          }
          uint32_t pkd[16];
#pragma unroll
          for (int v = 0; v < 16; ++v)
            pkd[v] = ptx::pack2<kBF16>(__uint_as_float(r[2 * v]), __uint_as_float(r[2 * v + 1]));
          if (row_ok && cc * 32 < args.dl && in_bounds(krow < kv_rows, kSiteBwdKV)) {
            uint4* dst = reinterpret_cast<uint4*>(row + cc * 64);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              dst[v] = make_uint4(pkd[4 * v], pkd[4 * v + 1], pkd[4 * v + 2], pkd[4 * v + 3]);
          }
        }
      };
      int i, it_idx = 0;
      while (it.next(i)) {
        if (it_idx++ == n_iters - 1) {
          // the unit's last dV MMA precedes its last dQ: take dV out first, so the next unit's dV can start
          ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_dv_done), ku & 1, args.budget_ns, abortp));
          if (!ok) break;
          ptx::tc_fence_after();
          epilogue(false);
        }
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_dq_full), gi & 1, args.budget_ns, abortp));
        if (!ok) break;
        ptx::tc_fence_after();
        const int row0 = (int)((size_t)u.bh * Npad + (size_t)i * kTile) + wq * 32;
        // one 32 x 32 fp32 box: staging buffer (after the previous box has been read out of it) -> TMA reduce-add
        auto reduce_box = [&](const uint32_t (&r)[32], int col) {
          if (lane == 0) ptx::bulk_wait_group_read<0>();
          __syncwarp();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(stage + lane * 128 + ((k ^ (lane & 7)) * 16)) =
                make_uint4(r[4 * k], r[4 * k + 1], r[4 * k + 2], r[4 * k + 3]);
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            // the 32 x 32 box lies inside the [BH * Npad][dl] accumulator
            if (in_bounds(row0 >= 0 && (size_t)row0 + 32 <= (size_t)args.BH * Npad && col + 32 <= args.dl, kSiteBwdDq))
              ptx::tma_reduce_add_2d(&map_dq, col, row0, stage_addr);
            ptx::bulk_commit_group();
          }
        };
        uint32_t ra[32], rb[32];
        ptx::tmem_ld32(tmem + lane_base + C::kColDQ, ra);
        ptx::tmem_ld32(tmem + lane_base + C::kColDQ + 32, rb);
        ptx::tmem_ld_wait();
        // boxes past the head dim (32 / 96 on the 64 / 128 kernels) hold only zeros and are not reduced
        if constexpr (D == 64) {
          ptx::tc_fence_before();
          ptx::mbar_arrive(ptx::smem_addr(&bar_dq_free));  // TMEM columns may now be overwritten
          reduce_box(ra, 0);
          if (32 < args.dl) reduce_box(rb, 32);
        } else {
          // d = 128: the columns are the next dP^T's, so all four chunks leave TMEM before any wait on the
          // staging buffer (registers hold up to three chunks)
          reduce_box(ra, 0);
          uint32_t rc[32], rd[32];
          ptx::tmem_ld32(tmem + lane_base + C::kColDQ + 64, rc);
          ptx::tmem_ld32(tmem + lane_base + C::kColDQ + 96, rd);
          ptx::tmem_ld_wait();
          ptx::tc_fence_before();
          ptx::mbar_arrive(ptx::smem_addr(&bar_dq_free));
          reduce_box(rb, 32);
          reduce_box(rc, 64);
          if (96 < args.dl) reduce_box(rd, 96);
        }
        ++gi;
      }
      if (!ok) break;
      // ---- dK of this unit (dV went out before the last dQ), or zeros for both when no query sees the keys
      if (n_iters > 0) {
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_done), ku & 1, args.budget_ns, abortp));
        if (!ok) break;
        ptx::tc_fence_after();
      } else {
        epilogue(false);
      }
      epilogue(true);
      if (n_iters > 0) ++ku;
    }
    if (lane == 0) ptx::bulk_wait_group<0>();  // all reductions performed before the CTA retires
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------------------------ idle warps 14, 15
#if FA_BWD_SETMAXNREG
    ptx::setmaxnreg_dec<kBwdRegsLow>();  // every warp of the MMA / TMA warpgroup takes the same budget
#endif
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------ host side
template <int D, bool BF>
cudaError_t launch_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                       const CUtensorMap& mdq,
                       const void* o, const void* dout, const float* lse, void* dq, const BwdArgs& a,
                       cudaStream_t st, cudaEvent_t ev_start, cudaEvent_t ev_stop) {
  using C = BwdCfg<D>;
  const int Npad = a.nT * kTile;
  const long long rows = (long long)a.BH * Npad;
  const long long pre_warps = (rows + (256 / D) - 1) / (256 / D);  // rows per warp pass: 4 (d=64) or 2 (d=128)
  const unsigned pre_blocks = (unsigned)std::min<long long>((pre_warps + 7) / 8, 148LL * 16);
  bwd_pre_kernel<D, BF><<<pre_blocks, 256, 0, st>>>(o, dout, lse, a.dq_acc, const_cast<float*>(a.lse2),
                                                     const_cast<float*>(a.Dv), a.N, Npad, rows, a.scale, a.cu_q,
                                                     a.total_q, a.H, a.dl);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> smem_set{0};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (!(smem_set.load() & (1ull << (dev & 63)))) {
    e = cudaFuncSetAttribute(bwd_kernel<D, BF>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    smem_set.fetch_or(1ull << (dev & 63));
  }
  // persistent: one CTA per SM at most (each walks its share of the units)
  int sms = 0;
  if ((e = device_sm_count(dev, &sms)) != cudaSuccess) return e;
  const long long units = (long long)a.nTk * a.BH;
  const unsigned grid = (unsigned)std::min<long long>(units, sms);
  if (ev_start && (e = cudaEventRecord(ev_start, st)) != cudaSuccess) return e;
  bwd_kernel<D, BF><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, mdo, mdq, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev_stop && (e = cudaEventRecord(ev_stop, st)) != cudaSuccess) return e;
  const long long total_vec8 = (long long)a.BH * (a.cu_q ? Npad : a.N) * a.dl / 8;
  const unsigned blocks = (unsigned)std::min<long long>((total_vec8 + 255) / 256, 148LL * 16);
  bwd_dq_kernel<D, BF><<<blocks, 256, 0, st>>>(a.dq_acc, dq, a.N, Npad, total_vec8, a.cu_q, a.total_q, a.H, a.dl);
  return cudaGetLastError();
}

}  // namespace fa
