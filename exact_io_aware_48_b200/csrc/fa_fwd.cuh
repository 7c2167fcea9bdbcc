// fa_fwd.cuh -- forward kernel: exact attention tile by tile with online softmax on sm_100a.
//
// Method (FlashAttention review page, "Method"; explainer page, "online softmax"; slide deck "Executable shape"):
// Q, K, V are cut into 128-row tiles; K/V tiles stream through shared memory past resident Q tiles; per row the
// running max m and denominator l are kept on chip and earlier partial outputs are rescaled when m grows; only O
// and the per-row logsumexp reach HBM.  The slide deck's loop runs K/V outer and Q inner with the state
// round-tripped per Q block; here the Q tiles stay resident (Q outer) so the state never leaves the chip -- the
// result is the same (online softmax is order independent in exact arithmetic).
//
// B200 mapping (one CTA = two 128-row Q tiles of one (b, h), 320 threads, one CTA per SM):
//   warp 9      TMA producer: Q tiles once, then K_j, V_j into a ring of shared-memory slots (mbarrier full/empty)
//   warp 8      MMA issuer (one thread): S_t = Q_t K_j^T into TMEM (fp32), O_t += P_t V_j with P_t read from TMEM
//   warps 0-3   softmax for Q tile 0, warps 4-7 for Q tile 1: each thread owns one query row (the TMEM 32x32b
//               access pattern hands a thread a whole row), so row max and row sum need no shuffles.
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,256+d), O_1 [256+d,256+2d); P_t (16-bit pairs)
// overwrites the first 64 columns of S_t after they have been read into registers.
// The two Q tiles ping-pong: while the softmax warps of one tile work, the tensor core runs the other tile's
// P V and next Q K^T.  Rescaling of O is lazy: a row's reference max only moves when the tile max exceeds it by
// more than 8 (log2 units), so O is read-modified-written in TMEM rarely; O / l stays exact in real arithmetic
// because acc and l always share the same reference max.
#pragma once
#include "fa_common.cuh"

namespace fa {

// kTiles = Q tiles per CTA.  2: one CTA per SM (320 threads, 512 TMEM columns), the two tiles ping-pong on the
// tensor core.  1: two CTAs per SM (192 threads, 256 TMEM columns, <= half the shared memory each), the two CTAs'
// chains interleave on the tensor core and the hardware schedules 128-row units (finer load balance).
template <int D, int kTiles = 2>
struct FwdCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(kTiles == 1 || kTiles == 2, "Q tiles per CTA");
  static constexpr int kSlotBytes = kTile * D * 2;  // one 128 x D tile of 16-bit values
  static constexpr int kSubTiles = D / 64;           // 128-byte-wide column blocks (one TMA box each)
  static constexpr int kNumSlots = kTiles == 2 ? (D == 128 ? 4 : 8) : (D == 128 ? 2 : 4);
  static constexpr int kQBytes = kTiles * kSlotBytes;
  static constexpr int kSmemBytes = kQBytes + kNumSlots * kSlotBytes + 1024;
  static constexpr int kWarpMma = 4 * kTiles, kWarpLoad = 4 * kTiles + 1;
  static constexpr int kThreads = 32 * (4 * kTiles + 2);
  static constexpr uint32_t kTmemCols = kTiles == 2 ? 512 : 256;
  static constexpr uint32_t kColO = 128 * kTiles;  // O_t at kColO + t * D
};

// Every kExpFmaEvery-th pair of probabilities is exponentiated on the FMA pipe (see ptx::exp2_fma); 0 = never.
// Measured on B200 (same box, interleaved runs): 1 pair in 16 gains 1-5% (GPT-2 shape 286 -> 299 TFLOP/s,
// N = 4096 800 -> 819, N = 16384 1109 -> 1122); 1 in 8 gains nothing (GPT-2 shape 4% slower) and 1 in 4 loses 6%.
#ifndef FA_FWD_EXP_FMA_EVERY
#define FA_FWD_EXP_FMA_EVERY 16
#endif
constexpr int kExpFmaEvery = FA_FWD_EXP_FMA_EVERY;

struct FwdArgs {
  void* o;
  float* lse;
  const int32_t* key_lens;
  const int32_t* row_ptr;  // CSR of the block mask (nullptr: dense)
  const int32_t* col_idx;
  long long list_head_stride;  // per-head masks: int32 distance between heads' lists (0: one mask for all heads)
  const int32_t* cu_q;  // packed variable-length batch: cumulative sequence lengths (nullptr: dense [B,H,N,d])
  const int32_t* cu_k;
  int total_q, total_k;  // packed: token counts; O is [total_q, H, d], LSE [H, total_q]
  int H, N, nT, npairs, BH;  // packed: N = the longest query sequence, Nk the longest key sequence
  int Nk;
  int dl;  // head dim of the tensors: D, or 32 / 96 run on the 64 / 128 kernels (TMA zero-fills the columns past dl)
  // split-K/V decode: the N queries of (b, h) are the last N positions of its sequence, so query r sees key c iff
  // c < len_k and (causal) c <= r + len_k - N; unit s of a Q tile covers K/V tiles [s*kv_split_tiles, ...+ that)
  int nsplit, kv_split_tiles;
  float* o_part;    // [nsplit][BH][128*nT][d] fp32: O of each split, normalised by its own l
  float* lse_part;  // [nsplit][BH][128*nT] fp32: natural-log LSE of each split, -inf if it saw no key
  int causal;
  float scale_log2;  // softmax_scale * log2(e)
  uint64_t budget_ns;
};

// One unit of work: kTiles consecutive 128-row Q tiles of one (b, h).  Units are ordered longest first (latest Q
// tiles first under the causal mask); the kernel is persistent and walks them with UnitSeq.
struct FwdUnit {
  int qt0, bh, h, kv_lim, end0, end1;
  int split, begin, off;  // split-K/V: split index, first K/V tile, causal offset (0 otherwise)
  SeqGeom g;
  bool has1;
};

constexpr int kModeDense = 0, kModePacked = 1, kModeSplit = 2;

template <int kMode>
__device__ __forceinline__ FwdUnit fwd_unit(int L, const FwdArgs& a, int tiles) {
  FwdUnit u;
  u.split = 0;
  if constexpr (kMode == kModeSplit) {  // units split-major: every split of every Q tile
    const int per = a.npairs * a.BH;
    u.split = L / per;
    L -= u.split * per;
  }
  const int pair = a.npairs - 1 - L / a.BH;
  u.bh = L % a.BH;
  u.h = u.bh % a.H;
  u.qt0 = tiles * pair;
  u.g = seq_geom(kMode == kModePacked ? a.cu_q : nullptr, a.cu_k, a.key_lens, u.bh / a.H, a.N, a.Nk, a.total_q,
                 a.total_k);
  if constexpr (kMode == kModeSplit) u.g.lk = key_limit(a.key_lens, u.bh / a.H, a.Nk);
  const int nTq = (u.g.lq + kTile - 1) / kTile;  // Q tiles of this sequence
  u.has1 = tiles == 2 && u.qt0 + 1 < nTq;
  u.kv_lim = u.g.lk;
  const bool causal = a.causal != 0;
  if constexpr (kMode == kModeSplit) {
    u.off = causal ? u.kv_lim - a.N : 0;
    u.begin = u.split * a.kv_split_tiles;
    const int stop = u.begin + a.kv_split_tiles;
    u.end0 = u.qt0 < nTq ? min(kv_tile_end_off(u.qt0, u.kv_lim, causal, u.off), stop) : 0;
    u.end1 = u.has1 ? min(kv_tile_end_off(u.qt0 + 1, u.kv_lim, causal, u.off), stop) : 0;
  } else {
    u.off = 0;
    u.begin = 0;
    u.end0 = u.qt0 < nTq ? kv_tile_end(u.qt0, u.kv_lim, causal) : 0;  // a tile past the sequence sees nothing
    u.end1 = u.has1 ? kv_tile_end(u.qt0 + 1, u.kv_lim, causal) : 0;
  }
  return u;
}

__device__ __forceinline__ void fwd_tiles(PairTileIter& it, const FwdUnit& u, const FwdArgs& a) {
  if (a.row_ptr != nullptr)
    it.init_sparse(a.row_ptr + u.h * a.list_head_stride, a.col_idx + u.h * a.list_head_stride, u.qt0, a.nT, u.end0,
                   u.end1);
  else
    it.init_dense(u.end0, u.end1, u.begin);
}

// kMode: kModeDense, kModePacked (packed variable-length batch, FwdArgs::cu_q set) or kModeSplit (split-K/V
// decode, partial results to o_part / lse_part); separate instantiations, so the dense kernels carry none of the
// other modes' state.
template <int D, bool kBF16, int kTiles, int kMode>
__global__ void __launch_bounds__(FwdCfg<D, kTiles>::kThreads, 3 - kTiles)
    fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
               const __grid_constant__ CUtensorMap map_v, const FwdArgs args) {
  using C = FwdCfg<D, kTiles>;
  constexpr int NS = C::kNumSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;

  // bar_sd[g % NSD]: every MMA of K/V step g (its S, and the previous step's P V) has completed.  K_g's slot was
  // last read in step g - NSD and V_g's slot in step g - NSD + 1 (V is read by the next step's P V), so the producer
  // waits for those; one commit per step releases both of a step's slots.
  constexpr int NSD = NS / 2;
  __shared__ __align__(8) uint64_t bar_q, bar_q_free, bar_full[NS], bar_sd[NSD], bar_s[2], bar_p[2], bar_o[2],
      bar_o_free[2], bar_drain;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  volatile int* abortp = &abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const bool causal = args.causal != 0;
  constexpr bool packed = kMode == kModePacked;
  constexpr bool split = kMode == kModeSplit;
  const int total_units = args.npairs * args.BH * (split ? args.nsplit : 1);

  if (threadIdx.x == 0) {
    ptx::mbar_init(ptx::smem_addr(&bar_q), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_q_free), 1);
    for (int s = 0; s < NS; ++s) ptx::mbar_init(ptx::smem_addr(&bar_full[s]), 1);
    for (int s = 0; s < NSD; ++s) ptx::mbar_init(ptx::smem_addr(&bar_sd[s]), 1);
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(ptx::smem_addr(&bar_s[t]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_p[t]), 128);
      ptx::mbar_init(ptx::smem_addr(&bar_o[t]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_o_free[t]), 128);
    }
    ptx::mbar_init(ptx::smem_addr(&bar_drain), 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == C::kWarpMma) {
    ptx::tmem_alloc(ptx::smem_addr(&tmem_base_sh), C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // Every role walks the same unit sequence and, per unit, the same K/V tile list; barrier phases and ring
  // positions run on across units.
  UnitSeq us;
  us.init(total_units);
  int L;

  if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tensormap(&map_q);
      ptx::prefetch_tensormap(&map_k);
      ptx::prefetch_tensormap(&map_v);
      const uint32_t bq = ptx::smem_addr(&bar_q);
      int n = 0, g = 0, ku = 0, j, fl;  // g: K/V steps loaded
      bool ok = true;
      while (ok && us.next(L)) {
        const FwdUnit u = fwd_unit<kMode>(L, args, kTiles);
        PairTileIter it;
        fwd_tiles(it, u, args);
        // the Q buffer is free once every S MMA of the previous unit has completed
        if (ku > 0 && !wait_or_abort(ptx::smem_addr(&bar_q_free), (ku - 1) & 1, args.budget_ns, abortp)) break;
        ptx::mbar_arrive_expect_tx(bq, (u.has1 ? 2 : 1) * C::kSlotBytes);
        for (int t = 0; t < (u.has1 ? 2 : 1); ++t)
          for (int c = 0; c < C::kSubTiles; ++c)
            tma_rows(ptx::smem_addr(sQ + t * C::kSlotBytes + c * 16384), &map_q, c, (u.qt0 + t) * kTile, u.g.q0, u.bh,
                     u.h, packed, bq);
        while (ok && it.next(j, fl)) {
          for (int kv = 0; kv < 2; ++kv) {
            const int s = n % NS;
            const int x = g - NSD + kv;  // the step that last read this slot
            if (x >= 0 && !wait_or_abort(ptx::smem_addr(&bar_sd[x % NSD]), (x / NSD) & 1, args.budget_ns, abortp)) {
              ok = false;
              break;
            }
            const uint32_t bf = ptx::smem_addr(&bar_full[s]);
            ptx::mbar_arrive_expect_tx(bf, C::kSlotBytes);
            const CUtensorMap* map = kv == 0 ? &map_k : &map_v;
            for (int c = 0; c < C::kSubTiles; ++c)
              tma_rows(ptx::smem_addr(sKV + s * C::kSlotBytes + c * 16384), map, c, j * kTile, u.g.k0, u.bh, u.h,
                       packed, bf);
            ++n;
          }
          ++g;
        }
        ++ku;
      }
      // Let every copy this thread issued land before the CTA can exit (immediate in the normal path).
      if (ku > 0) ptx::mbar_wait(bq, (ku - 1) & 1, args.budget_ns);
      for (int k = (n > NS ? n - NS : 0); k < n; ++k)
        ptx::mbar_wait(ptx::smem_addr(&bar_full[k % NS]), (k / NS) & 1, args.budget_ns);
    }
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_f16(kBF16, false, false, 128, 128);
      constexpr uint32_t idesc_o = ptx::idesc_f16(kBF16, false, true, 128, D);
      // descriptors built once and advanced by constants per MMA (one add each)
      const uint64_t dq0 = ptx::sw128_desc(ptx::smem_addr(sQ), 16, 1024);        // Q tiles, K-major
      const uint64_t dkv_k = ptx::sw128_desc(ptx::smem_addr(sKV), 16, 1024);     // K tiles, K-major
      const uint64_t dkv_mn = ptx::sw128_desc(ptx::smem_addr(sKV), 16384, 1024); // V tiles, M/N-major
      bool ok = true;
      int n = 0, g = 0, ku = 0, j, fl;  // g: K/V steps issued
      int pend_slot = 0, pend_flags = 0;
      uint32_t pend_phase = 0;
      uint32_t p_phase[2] = {0, 0};
      int pv_count[2] = {0, 0};

      // O_t += P_t V  (A = P_t from TMEM, B = V tile, M/N-major, 128-byte swizzle)
      auto issue_pv = [&](int t, int slot) {
        const uint64_t dv = ptx::desc_advance(dkv_mn, slot * C::kSlotBytes);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          ptx::mma_ts(tmem + C::kColO + t * D, tmem + t * 128 + kk * 8, ptx::desc_advance(dv, kk * 2048), idesc_o,
                      (pv_count[t] > 0 || kk > 0) ? 1u : 0u);
        ++pv_count[t];
      };
      // S_t = Q_t K^T  (both K-major, 128-byte swizzle, K = D in steps of 16)
      auto issue_s = [&](int t, int slot) {
        const uint64_t dqa = ptx::desc_advance(dq0, t * C::kSlotBytes);
        const uint64_t dkb = ptx::desc_advance(dkv_k, slot * C::kSlotBytes);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
          ptx::mma_ss(tmem + t * 128, ptx::desc_advance(dqa, off), ptx::desc_advance(dkb, off), idesc_s,
                      kk > 0 ? 1u : 0u);
        }
      };
      // Issue the pending P V of the previous visible tile for tile t (waits for its P).  The first P V of a unit
      // overwrites O_t, so it also waits until the epilogue has read the previous unit's O_t.
      bool v_ready = false;
      // `k_wait` (a K slot's barrier and phase, bar 0 = none) is waited for together with this P V's own waits, so
      // the MMA thread stops once rather than again before the next S: on sm_100a each wait of the issuing thread
      // lets its queued MMAs drain first.
      auto flush_pv = [&](int t, uint32_t k_bar = 0, uint32_t k_phase = 0) -> bool {
        if (!(pend_flags & (1 << t))) return true;
        if (!wait_or_abort(ptx::smem_addr(&bar_p[t]), p_phase[t], args.budget_ns, abortp)) return false;
        p_phase[t] ^= 1;
        if (!v_ready) {
          if (!wait_or_abort(ptx::smem_addr(&bar_full[pend_slot]), pend_phase, args.budget_ns, abortp)) return false;
          v_ready = true;
        }
        if (k_bar != 0 && !wait_or_abort(k_bar, k_phase, args.budget_ns, abortp)) return false;
        if (pv_count[t] == 0 && ku > 0 &&
            !wait_or_abort(ptx::smem_addr(&bar_o_free[t]), (ku - 1) & 1, args.budget_ns, abortp))
          return false;
        ptx::tc_fence_after();
        issue_pv(t, pend_slot);
        return true;
      };

      while (ok && us.next(L)) {
        const FwdUnit u = fwd_unit<kMode>(L, args, kTiles);
        PairTileIter it;
        fwd_tiles(it, u, args);
        if (!(ok = wait_or_abort(ptx::smem_addr(&bar_q), ku & 1, args.budget_ns, abortp))) break;
        ptx::tc_fence_after();
        pend_flags = 0;
        pv_count[0] = pv_count[1] = 0;
        v_ready = false;
        while (ok && it.next(j, fl)) {
          const int sK = n % NS;
          const uint32_t phK = (n / NS) & 1;
          ++n;
          const int sV = n % NS;
          const uint32_t phV = (n / NS) & 1;
          ++n;
          // K_j is waited for inside the first P V's waits when there is one before the first S (two-tile kernel;
          // measured slower in the one-tile kernel, whose K/V loads have less lead)
          bool k_ready = false;
          const int t_first = (fl & 1) ? 0 : 1;  // the first tile that sees K_j
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if (ok) {
              if (kTiles == 2 && t == t_first && !k_ready && (pend_flags & (1 << t))) {
                ok = flush_pv(t, ptx::smem_addr(&bar_full[sK]), phK);
                k_ready = ok;
              } else {
                ok = flush_pv(t);
              }
            }
            if (ok && (fl & (1 << t))) {
              if (!k_ready) {
                ok = wait_or_abort(ptx::smem_addr(&bar_full[sK]), phK, args.budget_ns, abortp);
                ptx::tc_fence_after();
                k_ready = true;
              }
              if (ok) {
                issue_s(t, sK);
                ptx::mma_commit(ptx::smem_addr(&bar_s[t]));
              }
            }
          }
          if (!ok) break;
          ptx::mma_commit(ptx::smem_addr(&bar_sd[g % NSD]));  // this K and the previous V consumed
          ++g;
          pend_slot = sV;
          pend_phase = phV;
          pend_flags = fl;
          v_ready = false;
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&bar_q_free));  // every S of this unit issued: Q may be replaced
#pragma unroll
        for (int t = 0; t < 2; ++t)
          if (ok) ok = flush_pv(t);
        if (!ok) break;
        // (this unit's last V is released by the next step's commit)
        // A tile that had no P V in this unit did not wait for the previous unit's epilogue; wait now, or two
        // back-to-back empty units would complete two phases of bar_o before its softmax warps look (ABA).
        for (int t = 0; t < kTiles && ok; ++t)
          if (pv_count[t] == 0 && ku > 0)
            ok = wait_or_abort(ptx::smem_addr(&bar_o_free[t]), (ku - 1) & 1, args.budget_ns, abortp);
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&bar_o[0]));
        ptx::mma_commit(ptx::smem_addr(&bar_o[1]));
        ++ku;
      }
      // No MMA may still be running when the tensor memory is released.
      ptx::mma_commit(ptx::smem_addr(&bar_drain));
      ptx::mbar_wait(ptx::smem_addr(&bar_drain), 0, args.budget_ns);
    }
  } else {
    // ------------------------------------------------------------------------------------------ softmax warps
    const int t = warp / 4;
    const int quarter = warp % 4;
    const int row = quarter * 32 + lane;  // row within the Q tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + t * 128;
    const uint32_t tO = tmem + lane_base + C::kColO + t * D;
    const float scale_log2 = args.scale_log2;
    uint32_t s_phase = 0;
    int ku = 0;
    bool ok = true;
    while (ok && us.next(L)) {
      FwdUnit u = fwd_unit<kMode>(L, args, kTiles);
      PairTileIter it;
      fwd_tiles(it, u, args);
      const int u_bh = u.bh;
      const bool u_has1 = u.has1;
      const int qt = u.qt0 + t;
      const int grow = qt * kTile + row;  // row within the sequence
      const int kv_lim = u.kv_lim;
      int coff = 0;  // split-K/V causal: keys c <= grow + coff
      if constexpr (split) coff = u.off;
      float m_ref = -INFINITY;
      ptx::f32x2 lacc[2] = {{0.f, 0.f}, {0.f, 0.f}};  // running denominator l, as four partial sums
      int kidx = 0;
      int j, fl;
      while (it.next(j, fl)) {
        if (!(fl & (1 << t))) continue;
        // every lane waits; the verdict is made warp-uniform before any warp-collective TMEM access
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_s[t]), s_phase, args.budget_ns, abortp));
        if (!ok) break;
        s_phase ^= 1;
        ptx::tc_fence_after();
        uint32_t sr[128];
        ptx::tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        ptx::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        ptx::tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        ptx::tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        ptx::tmem_ld_wait();
        float* s = reinterpret_cast<float*>(sr);
        // element masks only on tiles that straddle the diagonal or the key limit
        if constexpr (split) {
          if ((causal && (j + 1) * kTile - 1 > qt * kTile + coff) || (j + 1) * kTile > kv_lim) {
            const int c0 = j * kTile;
            const int lim = causal ? min(kv_lim, grow + 1 + coff) : kv_lim;  // keys c < lim are visible
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (c0 + i >= lim) s[i] = -INFINITY;
          }
        } else {
          if ((causal && j >= qt) || (j + 1) * kTile > kv_lim) {
            const int c0 = j * kTile;
            const int lim = causal ? min(kv_lim, grow + 1) : kv_lim;  // keys c < lim are visible
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (c0 + i >= lim) s[i] = -INFINITY;
          }
        }
        // row max: 8 independent partial maxima with 3-input max (two new elements per instruction), then a tree
        float pm[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) pm[a] = fmaxf(s[a], s[a + 8]);
#pragma unroll
        for (int i = 16; i < 128; i += 16)
#pragma unroll
          for (int a = 0; a < 8; ++a) pm[a] = ptx::max3(pm[a], s[i + a], s[i + 8 + a]);
        const float mx =
            ptx::max3(ptx::max3(pm[0], pm[1], pm[2]), ptx::max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
        const float m_tile = mx * scale_log2;
        const bool need = m_tile > m_ref + 8.0f;
        float alpha = 1.0f;
        if (need) {
          alpha = ptx::ex2(m_ref - m_tile);  // 0 when nothing was visible before
          m_ref = m_tile;
        }
        const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
        if (need) {  // the running partial sums follow the reference max
          lacc[0].x *= alpha; lacc[0].y *= alpha; lacc[1].x *= alpha; lacc[1].y *= alpha;
        }
        const ptx::f32x2 sc2{scale_log2, scale_log2}, nm2{-m_use, -m_use};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const ptx::f32x2 x = ptx::fma2({s[h * 64 + 2 * i], s[h * 64 + 2 * i + 1]}, sc2, nm2);
            // one pair in kExpFmaEvery goes through the FMA-pipe exp2 so the MUFU pipe is not the only exp unit
            const bool emu = kExpFmaEvery > 0 && (i % (kExpFmaEvery > 0 ? kExpFmaEvery : 1)) == kExpFmaEvery - 1;
            const float p0 = emu ? ptx::exp2_fma(x.x) : ptx::ex2(x.x);
            const float p1 = emu ? ptx::exp2_fma(x.y) : ptx::ex2(x.y);
            pk[i] = ptx::pack2<kBF16>(p0, p1);
            // l sums the rounded P that P V multiplies, so O stays a convex mix of V rows
            lacc[i & 1] = ptx::add2(lacc[i & 1], ptx::unpack2<kBF16>(pk[i]));
          }
          ptx::tmem_st32(tS + h * 32, pk);
        }
        // rescale the running output (only if some row of this warp moved its reference max)
        if (kidx > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t orr[32];
            ptx::tmem_ld32(tO + c * 32, orr);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            ptx::tmem_st32(tO + c * 32, orr);
          }
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&bar_p[t]));
        ++kidx;
      }
      if (!ok) break;
      // ---------------------------------------------------------------------------------------- epilogue
      // O_t is read out of TMEM and released to the next unit's first P V before it is normalised and stored.
      ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_o[t]), ku & 1, args.budget_ns, abortp));
      if (!ok) break;
      ptx::tc_fence_after();
      // packed: the unit is worked out again rather than kept in registers through the K/V loop (the softmax
      // warps are at their register limit and the packed unit carries more state)
      if constexpr (packed || split) {
        u = fwd_unit<kMode>(L, args, kTiles);
      } else {
        u.bh = u_bh;  // dense: only these two are needed below
        u.has1 = u_has1;
        u.g.lq = args.N;
      }
      const bool row_ok = grow < u.g.lq && (t == 0 || u.has1);
      const float l_sum = (lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y);
      const bool nonempty = l_sum > 0.f;
      const float inv = nonempty ? 1.0f / l_sum : 0.0f;
      // split-K/V: this split's normalised O (fp32) and LSE go to the partial buffers for the combine kernel
      size_t prow = 0;
      if constexpr (split) prow = ((size_t)u.split * args.BH + u.bh) * (size_t)(args.nT * kTile) + grow;
      const size_t orow_idx = packed ? (size_t)(u.g.q0 + grow) * args.H + u.h : (size_t)u.bh * args.N + grow;
      uint8_t* orow = reinterpret_cast<uint8_t*>(args.o) + orow_idx * args.dl * 2;
      // extents checked in FA_DEBUG builds: rows of O (and entries of LSE), rows of the split partials
      const size_t o_rows = packed ? (size_t)args.total_q * args.H : (size_t)args.BH * args.N;
      const size_t part_rows = (size_t)args.nsplit * args.BH * args.nT * kTile;
      (void)o_rows;
      (void)part_rows;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        ptx::tmem_ld32(tO + c * 32, orr);
        ptx::tmem_ld_wait();
        if (c == D / 32 - 1) {
          ptx::tc_fence_before();
          ptx::mbar_arrive(ptx::smem_addr(&bar_o_free[t]));
        }
        if constexpr (split) {
          if (row_ok && in_bounds(prow < part_rows, kSiteSplitPart)) {
            float4* dst = reinterpret_cast<float4*>(args.o_part + prow * D + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const float4 x = make_float4(__uint_as_float(orr[4 * v]), __uint_as_float(orr[4 * v + 1]),
                                           __uint_as_float(orr[4 * v + 2]), __uint_as_float(orr[4 * v + 3]));
              dst[v] = nonempty ? make_float4(x.x * inv, x.y * inv, x.z * inv, x.w * inv)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a = nonempty ? __uint_as_float(orr[2 * i]) * inv : 0.0f;
            const float bb = nonempty ? __uint_as_float(orr[2 * i + 1]) * inv : 0.0f;
            pk[i] = ptx::pack2<kBF16>(a, bb);
          }
          if (row_ok && c * 32 < args.dl && in_bounds(orow_idx < o_rows, kSiteFwdO)) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      }
      if (row_ok) {
        const float lse_v = nonempty ? (m_ref + __log2f(l_sum)) * 0.69314718055994530942f : -INFINITY;
        if constexpr (split) {
          if (in_bounds(prow < part_rows, kSiteSplitPart)) args.lse_part[prow] = lse_v;
        } else {
          const size_t li = packed ? (size_t)u.h * args.total_q + u.g.q0 + grow : (size_t)u.bh * args.N + grow;
          if (in_bounds(li < o_rows, kSiteFwdLse)) args.lse[li] = lse_v;
        }
      }
      ++ku;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kWarpMma) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------ split combine
// Merges the splits of a split-K/V forward (the online-softmax merge of the explainer page applied to whole
// partial results): with m = max_s LSE_s and w_s = exp(LSE_s - m),  O = sum_s w_s O_s / sum_s w_s,
// LSE = m + log sum_s w_s; all splits empty -> O = 0, LSE = -inf.  One warp per (b, h, query row); lane s holds
// split s's LSE (nsplit <= 32), each lane D/32 output columns.  Memory-bound and small.
template <int D, bool kBF16>
__global__ void __launch_bounds__(256) splitkv_combine_kernel(const float* __restrict__ o_part,
                                                              const float* __restrict__ lse_part,
                                                              void* __restrict__ o, float* __restrict__ lse,
                                                              int nsplit, int BH, int N, int Npad, int dl) {
  const int lane = threadIdx.x % 32;
  const long long rows = (long long)BH * N;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) / 32;
  for (long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / 32; r < rows; r += nwarps) {
    const long long bh = r / N;
    const int q = (int)(r % N);
    const size_t prow0 = (size_t)bh * Npad + q;  // row of split 0
    const size_t split_stride = (size_t)BH * Npad;
    const float ls = lane < nsplit ? lse_part[lane * split_stride + prow0] : -INFINITY;
    float m = ls;
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, k));
    const float w = (m == -INFINITY || ls == -INFINITY) ? 0.f : __expf(ls - m);
    float wsum = w;
#pragma unroll
    for (int k = 16; k > 0; k >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, k);
    constexpr int kCols = D / 32;  // columns per lane: lane * kCols .. + kCols - 1
    float acc[kCols];
#pragma unroll
    for (int c = 0; c < kCols; ++c) acc[c] = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const float ws = __shfl_sync(0xffffffffu, w, s);
      if (ws == 0.f) continue;
      const float* src = o_part + (s * split_stride + prow0) * D + lane * kCols;
#pragma unroll
      for (int c = 0; c < kCols; c += 2) {
        const float2 x = *reinterpret_cast<const float2*>(src + c);
        acc[c] = fmaf(ws, x.x, acc[c]);
        acc[c + 1] = fmaf(ws, x.y, acc[c + 1]);
      }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint32_t pk[kCols / 2];
#pragma unroll
    for (int c = 0; c < kCols; c += 2) pk[c / 2] = ptx::pack2<kBF16>(acc[c] * inv, acc[c + 1] * inv);
    uint16_t* dst = reinterpret_cast<uint16_t*>(o) + ((size_t)bh * N + q) * dl + lane * kCols;
    if (lane * kCols < dl) {  // columns past the head dim are the zero padding
      if constexpr (kCols == 8) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      } else if constexpr (kCols == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(pk[0], pk[1]);
      } else {
        *reinterpret_cast<uint32_t*>(dst) = pk[0];
      }
    }
    if (lane == 0) lse[(size_t)bh * N + q] = wsum > 0.f ? m + __logf(wsum) : -INFINITY;
  }
}

}  // namespace fa
