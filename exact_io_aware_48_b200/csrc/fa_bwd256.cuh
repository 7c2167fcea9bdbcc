// fa_bwd256.cuh -- backward main kernel for head dim 256 (sm_100a), and the backward's host-side dispatch.
//
// Same method and gradients as fa_bwd.cuh (FlashAttention review page, claim C7 / E-recompute: P recomputed tile by
// tile from the saved logsumexp, the N x N matrix never in HBM):
//     P = exp(scale * Q K^T - LSE),  dV = P^T dO,  dS = P * (dO V^T - D),  dQ = scale * dS K,  dK = scale * dS^T Q.
//
// At d = 256 one 128 x 256 16-bit tile is 64 KB, so the d = 64 / 128 layout (K, V resident per key tile, Q and dO
// streamed as whole tiles, dK and dV accumulating in TMEM) fits neither shared memory nor TMEM: dK and dV alone
// would take all 512 TMEM columns.  This kernel keeps the d = 128 kernel's roles and TMEM map and changes two things:
//   * Two passes over halves of the head dimension.  A unit is (key tile j, half h, head): it recomputes S^T and
//     dP^T over the full d = 256 and accumulates only dV[:, half h] and dK[:, half h] in TMEM (128 columns each),
//     and sends dQ[:, half h] = scale * dS K[:, half h] to the fp32 accumulator.  The two passes together give every
//     column once; S^T and dP^T are computed twice (29.4 instead of 21 MFLOP of products per tile pair and pass
//     pair: 5/7 of the work is the algorithmic 2.5x forward).
//   * The key tile K_j (four 16 KB boxes of 128 rows x 64 columns) stays resident for the unit: it is the A operand
//     of every S^T and the B operand of every dQ_h.  Every other operand streams through one ring of 16 KB boxes in
//     exactly the order the MMA thread consumes them, and each box is released after its single use, so no box is
//     ever held while later ones wait for its slot.  Per Q tile i of a unit:
//         S^T  : Q box c for c = 0..3 (A = resident K box c)   4 boxes, contraction over d in four steps of 64
//         dP^T : (V box c, dO box c) for c = 0..3             8 boxes
//         dV_h : dO boxes 2h, 2h+1                            2 boxes, one N = 128 operand
//         dQ_h : (resident K boxes 2h, 2h+1)                  0 boxes
//         dK_h : Q boxes 2h, 2h+1                             2 boxes
//     in the MMA order S^T_first, then per i: dP^T_i [P^T_i] dV_i, S^T_{i+1} [dS^T_i] dQ_i, dK_i.  Every pair starts
//     at an even box position and the ring has an even number of slots, so the two boxes of a pair always sit in
//     adjacent slots 16 KB apart (the N-chunk stride of their shared-memory descriptor).  The next unit's K waits
//     until every MMA of the current unit has completed.
//   The LSE2 / D rows of each Q tile come through a separate two-entry ring.
// TMEM (512 columns): S^T [0,128); dP^T [128,256); dV_h [256,384); dK_h [384,512); P^T (16-bit pairs) over the S^T
// columns it replaces ([0,32) and [64,96)); dQ_h in the dP^T columns once they have been read.
#pragma once
#include "fa_bwd.cuh"

namespace fa {

struct Bwd256Cfg {
  static constexpr int D = 256;
  static constexpr int kHalf = 128;                    // head-dim columns per pass
  static constexpr int kBoxBytes = kTile * 64 * 2;     // 16 KB: 128 rows x 64 columns
  static constexpr int kBoxes = D / 64;                // column boxes of a 128 x 256 tile
  static constexpr int kKBytes = 4 * kTile * 64 * 2;   // resident K tile: four boxes
  static constexpr int kNumSlots = 6;                  // even, so a box pair never wraps around the ring
  static constexpr int kLdSlots = 2;                   // LSE2 / D rows of a Q tile, 1 KB each
  static constexpr int kDsBytes = kTile * kTile * 2;   // dS^T, 128 keys x 128 queries
  static constexpr int kStageBytes = 4 * 4096;         // dQ staging: one 32 x 32 fp32 box per drain warp
  static constexpr int kSmemBytes = kKBytes + kNumSlots * kBoxBytes + kDsBytes + kStageBytes + kLdSlots * 1024 + 1024;
  static constexpr int kThreads = 512;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384, kColDQ = 128;
  static constexpr uint32_t kColPT = 0, kPtHalf = 64;  // P^T of query half g at kColPT + kPtHalf * g
  static_assert(kNumSlots % 2 == 0, "box pairs must not wrap around the ring");
  static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

template <bool kBF16>
__global__ void __launch_bounds__(512, 1)
    bwd256_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_do,
                  const __grid_constant__ CUtensorMap map_dq, const BwdArgs args) {
  using C = Bwd256Cfg;
  constexpr int NS = C::kNumSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;
  uint8_t* sRing = sK + C::kKBytes;
  uint8_t* sDS = sRing + NS * C::kBoxBytes;
  uint8_t* sStage = sDS + C::kDsBytes;
  uint8_t* sLd = sStage + C::kStageBytes;

  __shared__ __align__(8) uint64_t bar_full[NS], bar_empty[NS], bar_ld_full[C::kLdSlots], bar_ld_empty[C::kLdSlots],
      bar_s, bar_dp, bar_p, bar_ds, bar_dq_full, bar_dq_free, bar_ds_free, bar_dv_done, bar_done, bar_dv_free,
      bar_dk_free, bar_drain, bar_kfull, bar_kfree;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_flag;
  volatile int* abortp = &abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int kWarpDrain = 8, kWarpMma = 12, kWarpLoad = 13;
  const bool causal = args.causal != 0;
  const int Npad = args.nT * kTile;
  const int total_units = args.nTk * 2 * args.BH;
  const bool packed = args.cu_q != nullptr;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(ptx::smem_addr(&bar_full[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_empty[s]), 1);
    }
    for (int s = 0; s < C::kLdSlots; ++s) {
      ptx::mbar_init(ptx::smem_addr(&bar_ld_full[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_ld_empty[s]), 256);
    }
    ptx::mbar_init(ptx::smem_addr(&bar_s), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dp), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_p), 256);
    ptx::mbar_init(ptx::smem_addr(&bar_ds), 256);
    ptx::mbar_init(ptx::smem_addr(&bar_dq_full), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dq_free), 128);
    ptx::mbar_init(ptx::smem_addr(&bar_ds_free), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dv_done), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_done), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_dv_free), 128);
    ptx::mbar_init(ptx::smem_addr(&bar_dk_free), 128);
    ptx::mbar_init(ptx::smem_addr(&bar_drain), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_kfull), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_kfree), 1);
    abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == kWarpMma) {
    ptx::tmem_alloc(ptx::smem_addr(&tmem_base_sh), C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = tmem_base_sh;

  // Unit L: key tile j = L / (2 BH) (longest causal columns first), then half h, then head.  Every role walks the
  // same unit sequence and, per unit, the same Q-tile list; box, Q-tile and unit counters run on across units.
  auto unit_of = [&](int L, int& half) {
    const int per = 2 * args.BH;
    const int j = L / per, r = L % per;
    half = r / args.BH;
    return bwd_unit(j * args.BH + r % args.BH, args);
  };
  auto tiles_of = [&](ColTileIter& it, const BwdUnit& u) {
    it.init(args.col_ptr ? args.col_ptr + u.h * args.list_head_stride : nullptr,
            args.row_idx + u.h * args.list_head_stride, u.j, u.nTq, causal ? u.j : 0, u.visible);
  };
  UnitSeq us;
  us.init(total_units);
  int L;

  if (warp == kWarpLoad) {
    // ------------------------------------------------------------------------------------------ TMA producer
#if FA_BWD_SETMAXNREG
    ptx::setmaxnreg_dec<512 - 128 - 2 * FA_BWD_REGS_HIGH>();
#endif
    if (lane == 0) {
      ptx::prefetch_tensormap(&map_q);
      ptx::prefetch_tensormap(&map_do);
      ptx::prefetch_tensormap(&map_k);
      ptx::prefetch_tensormap(&map_v);
      int nb = 0, gl = 0, ku = 0;
      bool ok = true;
      while (ok && us.next(L)) {
        int half;
        const BwdUnit u = unit_of(L, half);
        ColTileIter it;
        tiles_of(it, u);
        if (it.count() == 0) continue;
        // one 16 KB box (column box c, 128 rows from `row`) into the next ring slot
        auto box = [&](const CUtensorMap* map, int c, int row, int base) -> bool {
          const int s = nb % NS;
          if (!wait_or_abort(ptx::smem_addr(&bar_empty[s]), ((nb / NS) & 1) ^ 1, args.budget_ns, abortp)) return false;
          const uint32_t bf = ptx::smem_addr(&bar_full[s]);
          ptx::mbar_arrive_expect_tx(bf, C::kBoxBytes);
          tma_rows(ptx::smem_addr(sRing + s * C::kBoxBytes), map, c, row, base, u.bh, u.h, packed, bf);
          ++nb;
          return true;
        };
        // LSE2 / D rows of Q tile i into the next entry of their ring
        auto ld_rows = [&](int i) -> bool {
          const int s = gl % C::kLdSlots;
          if (!wait_or_abort(ptx::smem_addr(&bar_ld_empty[s]), ((gl / C::kLdSlots) & 1) ^ 1, args.budget_ns, abortp))
            return false;
          const uint32_t bf = ptx::smem_addr(&bar_ld_full[s]);
          const size_t row0 = (size_t)u.bh * Npad + (size_t)i * kTile;
          // the 128 rows lie inside the [BH][Npad] arrays (a skipped load is left out of the byte count)
          const bool side_ok = in_bounds(row0 + kTile <= (size_t)args.BH * Npad, kSiteBwdSide);
          ptx::mbar_arrive_expect_tx(bf, side_ok ? 1024 : 0);
          if (side_ok) {
            ptx::bulk_load(ptx::smem_addr(sLd + s * 1024), args.lse2 + row0, 512, bf);
            ptx::bulk_load(ptx::smem_addr(sLd + s * 1024 + 512), args.Dv + row0, 512, bf);
          }
          ++gl;
          return true;
        };
        auto scores = [&](const CUtensorMap* ma, int ra, int ba, const CUtensorMap* mb, int rb, int bb) -> bool {
          for (int c = 0; c < C::kBoxes; ++c)
            if (!box(ma, c, ra, ba) || !box(mb, c, rb, bb)) return false;
          return true;
        };
        auto qboxes = [&](int row, int base) -> bool {  // the four Q boxes of one S^T (K is resident)
          for (int c = 0; c < C::kBoxes; ++c)
            if (!box(&map_q, c, row, base)) return false;
          return true;
        };
        auto pair = [&](const CUtensorMap* m, int row, int base) -> bool {
          return box(m, 2 * half, row, base) && box(m, 2 * half + 1, row, base);
        };
        const int krow = u.j * kTile;
        int i, inext;
        bool have = it.next(i);
        ok = ld_rows(i) && qboxes(i * kTile, u.g.q0);
        // the resident K tile, once every MMA of the previous unit has completed (the first Q boxes are already
        // on their way, so the MMA pipe only waits for K itself)
        if (ok && ku > 0) ok = wait_or_abort(ptx::smem_addr(&bar_kfree), (ku - 1) & 1, args.budget_ns, abortp);
        if (ok) {
          const uint32_t bk = ptx::smem_addr(&bar_kfull);
          ptx::mbar_arrive_expect_tx(bk, C::kKBytes);
          for (int c = 0; c < C::kBoxes; ++c)
            tma_rows(ptx::smem_addr(sK + c * C::kBoxBytes), &map_k, c, krow, u.g.k0, u.bh, u.h, packed, bk);
          ++ku;
        }
        while (ok && have) {
          const bool have_next = it.next(inext);
          ok = scores(&map_v, krow, u.g.k0, &map_do, i * kTile, u.g.q0) && pair(&map_do, i * kTile, u.g.q0);
          if (ok && have_next) ok = ld_rows(inext) && qboxes(inext * kTile, u.g.q0);
          if (ok) ok = pair(&map_q, i * kTile, u.g.q0);
          have = have_next;
          i = inext;
        }
      }
      // Let every copy this thread issued land before the CTA can exit (immediate in the normal path).
      for (int k = (nb > NS ? nb - NS : 0); k < nb; ++k)
        ptx::mbar_wait(ptx::smem_addr(&bar_full[k % NS]), (k / NS) & 1, args.budget_ns);
      for (int k = (gl > C::kLdSlots ? gl - C::kLdSlots : 0); k < gl; ++k)
        ptx::mbar_wait(ptx::smem_addr(&bar_ld_full[k % C::kLdSlots]), (k / C::kLdSlots) & 1, args.budget_ns);
      if (ku > 0) ptx::mbar_wait(ptx::smem_addr(&bar_kfull), (ku - 1) & 1, args.budget_ns);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------------------------------ MMA issuer
#if FA_BWD_SETMAXNREG
    ptx::setmaxnreg_dec<512 - 128 - 2 * FA_BWD_REGS_HIGH>();
#endif
    if (lane == 0) {
      constexpr uint32_t id_sq = ptx::idesc_f16(kBF16, false, false, 128, 128);  // S^T, dP^T
      constexpr uint32_t id_dv = ptx::idesc_f16(kBF16, false, true, 128, C::kHalf);  // dV (A from TMEM), dK
      constexpr uint32_t id_dq = ptx::idesc_f16(kBF16, true, true, 128, C::kHalf);   // dQ
      const uint64_t dds_k = ptx::sw128_desc(ptx::smem_addr(sDS), 16, 1024);      // dS^T, K-major (dK)
      const uint64_t dds_mn = ptx::sw128_desc(ptx::smem_addr(sDS), 16384, 1024);  // dS, M-major (dQ)
      const uint64_t ring_k = ptx::sw128_desc(ptx::smem_addr(sRing), 16, 1024);   // a box, K-major
      const uint64_t k_k = ptx::sw128_desc(ptx::smem_addr(sK), 16, 1024);         // resident K box, K-major
      // a box pair (adjacent slots), M/N-major: 64-element N chunks one slot (16 KB) apart
      const uint64_t ring_mn = ptx::sw128_desc(ptx::smem_addr(sRing), C::kBoxBytes, 1024);
      constexpr auto kstep = [](int kk) { return (uint32_t)((kk / 4) * 16384 + (kk % 4) * 32); };
      int nb = 0;
      auto take = [&](int k) -> bool {  // wait until box k has landed
        if (!wait_or_abort(ptx::smem_addr(&bar_full[k % NS]), (k / NS) & 1, args.budget_ns, abortp)) return false;
        ptx::tc_fence_after();
        return true;
      };
      // boxes k .. k+count-1, all waited for before any of their MMAs is issued: on sm_100a each wait of the
      // issuing thread lets its queued MMAs drain first, so the waits of a group of MMAs are made back to back
      auto take_n = [&](int k, int count) -> bool {
        for (int i = 0; i < count; ++i)
          if (!wait_or_abort(ptx::smem_addr(&bar_full[(k + i) % NS]), ((k + i) / NS) & 1, args.budget_ns, abortp))
            return false;
        ptx::tc_fence_after();
        return true;
      };
      auto release = [&](int k) { ptx::mma_commit(ptx::smem_addr(&bar_empty[k % NS])); };
      auto off = [&](int k) { return (uint32_t)((k % NS) * C::kBoxBytes); };
      // S^T = K Q^T or dP^T = V dO^T over d = 256: four (A box, B box) pairs, both K-major
      // (two chunks, four boxes, per group: the ring holds six)
      auto scores = [&](uint32_t col, uint64_t& bar) -> bool {
        for (int c = 0; c < C::kBoxes; ++c) {
          if ((c & 1) == 0 && !take_n(nb, 4)) return false;
          const uint64_t da = ptx::desc_advance(ring_k, off(nb)), db = ptx::desc_advance(ring_k, off(nb + 1));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_ss(tmem + col, ptx::desc_advance(da, kk * 32), ptx::desc_advance(db, kk * 32), id_sq,
                        (c > 0 || kk > 0) ? 1u : 0u);
          release(nb);
          release(nb + 1);
          nb += 2;
        }
        ptx::mma_commit(ptx::smem_addr(&bar));
        return true;
      };
      // S^T = K Q^T over d = 256: A = resident K box c, B = the next ring box (Q box c), both K-major
      auto scores_k = [&]() -> bool {
        if (!take_n(nb, C::kBoxes)) return false;
        for (int c = 0; c < C::kBoxes; ++c) {
          const uint64_t da = ptx::desc_advance(k_k, c * C::kBoxBytes), db = ptx::desc_advance(ring_k, off(nb));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_ss(tmem + C::kColS, ptx::desc_advance(da, kk * 32), ptx::desc_advance(db, kk * 32), id_sq,
                        (c > 0 || kk > 0) ? 1u : 0u);
          release(nb);
          nb += 1;
        }
        ptx::mma_commit(ptx::smem_addr(&bar_s));
        return true;
      };
      // dV_h += P^T dO[:, h]  (P^T from TMEM, the dO pair as one N = 128 M/N-major operand)
      auto issue_dv = [&](bool first) -> bool {
        if (!take(nb) || !take(nb + 1)) return false;
        const uint64_t db = ptx::desc_advance(ring_mn, off(nb));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          ptx::mma_ts(tmem + C::kColDV, tmem + C::kColPT + (kk / 4) * C::kPtHalf + (kk % 4) * 8,
                      ptx::desc_advance(db, kk * 2048), id_dv, (!first || kk > 0) ? 1u : 0u);
        release(nb);
        release(nb + 1);
        nb += 2;
        return true;
      };
      // dQ_h = dS K[:, h]  (dS read M-major from the dS^T tile; resident K boxes 2h, 2h+1 as one N = 128 operand)
      auto issue_dq = [&](int half) {
        const uint64_t db =
            ptx::desc_advance(ptx::sw128_desc(ptx::smem_addr(sK), C::kBoxBytes, 1024), 2 * half * C::kBoxBytes);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          ptx::mma_ss(tmem + C::kColDQ, ptx::desc_advance(dds_mn, kk * 2048), ptx::desc_advance(db, kk * 2048), id_dq,
                      kk > 0 ? 1u : 0u);
        ptx::mma_commit(ptx::smem_addr(&bar_dq_full));
      };
      // dK_h += dS^T Q[:, h]  (dS^T K-major, the Q pair as one N = 128 operand)
      // (the caller has taken the pair, together with the dS^T wait)
      auto issue_dk = [&](bool first) {
        const uint64_t db = ptx::desc_advance(ring_mn, off(nb));
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          ptx::mma_ss(tmem + C::kColDK, ptx::desc_advance(dds_k, kstep(kk)), ptx::desc_advance(db, kk * 2048), id_dv,
                      (!first || kk > 0) ? 1u : 0u);
        release(nb);
        release(nb + 1);
        nb += 2;
      };
      int gi = 0, ku = 0;  // Q tiles and non-empty units processed so far
      bool ok = true;
      while (ok && us.next(L)) {
        int half;
        const BwdUnit u = unit_of(L, half);
        ColTileIter it;
        tiles_of(it, u);
        if (it.count() == 0) continue;
        auto acc_ready = [&](uint64_t& bar_free) -> bool {
          if (ku == 0) return true;
          if (!wait_or_abort(ptx::smem_addr(&bar_free), (ku - 1) & 1, args.budget_ns, abortp)) return false;
          ptx::tc_fence_after();
          return true;
        };
        int i, li = 0;
        bool have = it.next(i);
        if (!(ok = wait_or_abort(ptx::smem_addr(&bar_kfull), ku & 1, args.budget_ns, abortp))) break;
        ptx::tc_fence_after();
        if (!(ok = scores_k())) break;
        while (ok && have) {
          const uint32_t ph = gi & 1, ph_prev = (gi - 1) & 1;
          // dP^T_i lands in the columns that held dQ_{i-1}: wait until the drain warps have read it
          if (gi > 0 && !(ok = wait_or_abort(ptx::smem_addr(&bar_dq_free), ph_prev, args.budget_ns, abortp))) break;
          ptx::tc_fence_after();
          if (!(ok = scores(C::kColDP, bar_dp))) break;
          if (!(ok = wait_or_abort(ptx::smem_addr(&bar_p), ph, args.budget_ns, abortp))) break;
          ptx::tc_fence_after();
          if (li == 0 && !(ok = acc_ready(bar_dv_free))) break;
          if (!(ok = issue_dv(li == 0))) break;
          int inext;
          const bool have_next = it.next(inext);
          if (!have_next) ptx::mma_commit(ptx::smem_addr(&bar_dv_done));  // this unit's dV_h is final
          // S^T_{i+1} overwrites P^T_i only after dV_i has read it (MMAs complete in issue order)
          if (have_next && !(ok = scores_k())) break;
          // dS^T_i, dK_h's Q pair and (first tile) the dK accumulator: all waited for before dQ_i and dK_i
          if (!(ok = wait_or_abort(ptx::smem_addr(&bar_ds), ph, args.budget_ns, abortp))) break;
          if (!(ok = take_n(nb, 2))) break;
          if (li == 0 && !(ok = acc_ready(bar_dk_free))) break;
          ptx::tc_fence_after();
          issue_dq(half);
          issue_dk(li == 0);
          ptx::mma_commit(ptx::smem_addr(&bar_ds_free));
          ++gi;
          ++li;
          have = have_next;
          i = inext;
        }
        if (!ok) break;
        ptx::mma_commit(ptx::smem_addr(&bar_done));   // dK_h of this unit is final (and every MMA before it)
        ptx::mma_commit(ptx::smem_addr(&bar_kfree));  // the resident K tile is no longer read
        ++ku;
      }
      ptx::mma_commit(ptx::smem_addr(&bar_drain));
      ptx::mbar_wait(ptx::smem_addr(&bar_drain), 0, args.budget_ns);
    }
  } else if (warp < kWarpDrain) {
    // ------------------------------------------------------------------------------------------ P^T / dS^T warps
    // As at d = 128: warpgroup g handles queries [64g, 64g+64) of every key row (thread = key row = TMEM lane).
#if FA_BWD_SETMAXNREG
    ptx::setmaxnreg_inc<FA_BWD_REGS_HIGH>();
#endif
    const int g = warp / 4, quarter = warp % 4;
    const int c = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const ptx::f32x2 sl2v{args.scale_log2, args.scale_log2}, sc2{args.scale, args.scale};
    int gi = 0;
    bool ok = true;
    while (ok && us.next(L)) {
      int half;
      const BwdUnit u = unit_of(L, half);
      ColTileIter it;
      tiles_of(it, u);
      const int j = u.j, kv_lim = u.kv_lim;
      const int gc = j * kTile + c;
      int i;
      while (it.next(i)) {
        const int ls = gi % C::kLdSlots;
        const float* nlse2 = reinterpret_cast<const float*>(sLd + ls * 1024) + 64 * g;
        const float* nDrow = nlse2 + 128;
        const uint32_t ph = gi & 1;
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_ld_full[ls]), (gi / C::kLdSlots) & 1,
                                                    args.budget_ns, abortp));
        if (ok) ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_s), ph, args.budget_ns, abortp));
        if (!ok) break;
        ptx::tc_fence_after();
        const bool masked = (causal && i == j) || (j + 1) * kTile > kv_lim;
        const int rmin = causal ? gc - i * kTile - 64 * g : 0;
        const bool key_ok = gc < kv_lim;
        uint32_t pk[32];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t sr[32];
          ptx::tmem_ld32(tmem + lane_base + C::kColS + 64 * g + 32 * hh, sr);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const int r0 = 32 * hh + 2 * v;
            const float4 nl4 = *reinterpret_cast<const float4*>(nlse2 + (r0 & ~3));
            const ptx::f32x2 nl = (v & 1) ? ptx::f32x2{nl4.z, nl4.w} : ptx::f32x2{nl4.x, nl4.y};
            const ptx::f32x2 x =
                ptx::fma2({__uint_as_float(sr[2 * v]), __uint_as_float(sr[2 * v + 1])}, sl2v, nl);
            float p0 = ptx::ex2(x.x);
            float p1 = ptx::ex2(x.y);
            if (masked) {
              if (!key_ok || r0 < rmin) p0 = 0.f;
              if (!key_ok || r0 + 1 < rmin) p1 = 0.f;
            }
            pk[16 * hh + v] = ptx::pack2<kBF16>(p0, p1);
          }
        }
        // P^T of this half into the S^T columns this warpgroup has just read
        ptx::tmem_st32(tmem + lane_base + C::kColPT + C::kPtHalf * g, pk);
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&bar_p));
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_dp), ph, args.budget_ns, abortp));
        if (ok && gi > 0)
          ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_ds_free), (gi - 1) & 1, args.budget_ns,
                                                      abortp));
        if (!ok) break;
        ptx::tc_fence_after();
        uint8_t* rowp = sDS + g * 16384 + c * 128;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t dr[32];
          ptx::tmem_ld32(tmem + lane_base + C::kColDP + 64 * g + 32 * hh, dr);
          ptx::tmem_ld_wait();
          uint32_t o[16];
#pragma unroll
          for (int v = 0; v < 16; ++v) {
            const int r0 = 32 * hh + 2 * v;
            const float4 nd4 = *reinterpret_cast<const float4*>(nDrow + (r0 & ~3));
            const ptx::f32x2 nd = (v & 1) ? ptx::f32x2{nd4.z, nd4.w} : ptx::f32x2{nd4.x, nd4.y};
            const ptx::f32x2 t =
                ptx::fma2({__uint_as_float(dr[2 * v]), __uint_as_float(dr[2 * v + 1])}, sc2, nd);
            const ptx::f32x2 ds = ptx::mul2(ptx::unpack2<kBF16>(pk[16 * hh + v]), t);
            o[v] = ptx::pack2<kBF16>(ds.x, ds.y);
          }
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            const int chunk = (4 * hh + v) ^ (c & 7);
            *reinterpret_cast<uint4*>(rowp + chunk * 16) =
                make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
          }
        }
        ptx::fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&bar_ds));
        ptx::mbar_arrive(ptx::smem_addr(&bar_ld_empty[ls]));  // this Q tile's LSE2 / D rows are no longer read
        ++gi;
      }
    }
  } else if (warp < kWarpMma) {
    // ------------------------------------------------------------------------------------------ drain warps
    // dQ_h (thread = query row): 128 columns out of TMEM, 32 x 32 fp32 boxes through the staging buffer, TMA
    // reduce-add into dq_acc[:, 128h + ...].  dK_h, dV_h epilogue (thread = key row): columns [128h, 128h + 128).
    const int wq = warp - kWarpDrain;
    const uint32_t lane_base = static_cast<uint32_t>(wq * 32) << 16;
    uint8_t* stage = sStage + wq * 4096;
    const uint32_t stage_addr = ptx::smem_addr(stage);
    int gi = 0, ku = 0;
    bool ok = true;
    while (ok && us.next(L)) {
      int half;
      const BwdUnit u = unit_of(L, half);
      ColTileIter it;
      tiles_of(it, u);
      const int n_iters = it.count();
      const int gc = u.j * kTile + wq * 32 + lane;
      const bool row_ok = packed ? gc < u.g.lk : gc < args.N;
      const size_t krow = packed ? (size_t)(u.g.k0 + gc) * args.H + u.h : (size_t)u.bh * args.N + gc;
      const size_t kv_rows = packed ? (size_t)args.total_k * args.H : (size_t)args.BH * args.N;  // rows of dK, dV
      (void)kv_rows;
      auto epilogue = [&](bool is_dk) {
        uint8_t* row = reinterpret_cast<uint8_t*>(is_dk ? args.dk : args.dv) + krow * args.dl * 2 + half * C::kHalf * 2;
#pragma unroll 1
        for (int cc = 0; cc < C::kHalf / 32; ++cc) {
          uint32_t r[32];
          if (n_iters > 0) {
            ptx::tmem_ld32(tmem + lane_base + (is_dk ? C::kColDK : C::kColDV) + cc * 32, r);
            ptx::tmem_ld_wait();
            if (cc == C::kHalf / 32 - 1) {
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
          if (row_ok && in_bounds(krow < kv_rows, kSiteBwdKV)) {
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
          ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_dv_done), ku & 1, args.budget_ns, abortp));
          if (!ok) break;
          ptx::tc_fence_after();
          epilogue(false);
        }
        ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_dq_full), gi & 1, args.budget_ns, abortp));
        if (!ok) break;
        ptx::tc_fence_after();
        const int row0 = (int)((size_t)u.bh * Npad + (size_t)i * kTile) + wq * 32;
        const int col0 = half * C::kHalf;
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
            if (in_bounds(row0 >= 0 && (size_t)row0 + 32 <= (size_t)args.BH * Npad && col0 + col + 32 <= args.dl,
                          kSiteBwdDq))
              ptx::tma_reduce_add_2d(&map_dq, col0 + col, row0, stage_addr);
            ptx::bulk_commit_group();
          }
        };
        // at most two 32-column chunks in registers at a time (three spilled at this kernel's register budget)
        uint32_t ra[32], rb[32];
        ptx::tmem_ld32(tmem + lane_base + C::kColDQ, ra);
        ptx::tmem_ld32(tmem + lane_base + C::kColDQ + 32, rb);
        ptx::tmem_ld_wait();
        reduce_box(ra, 0);
        ptx::tmem_ld32(tmem + lane_base + C::kColDQ + 64, ra);
        ptx::tmem_ld_wait();
        reduce_box(rb, 32);
        ptx::tmem_ld32(tmem + lane_base + C::kColDQ + 96, rb);
        ptx::tmem_ld_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&bar_dq_free));  // the next dP^T may overwrite these columns
        reduce_box(ra, 64);
        reduce_box(rb, 96);
        ++gi;
      }
      if (!ok) break;
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
    ptx::setmaxnreg_dec<512 - 128 - 2 * FA_BWD_REGS_HIGH>();
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
template <bool BF>
cudaError_t launch_bwd256(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                          const CUtensorMap& mdo, const CUtensorMap& mdq, const void* o, const void* dout,
                          const float* lse, void* dq, const BwdArgs& a, cudaStream_t st, cudaEvent_t ev_start,
                          cudaEvent_t ev_stop) {
  using C = Bwd256Cfg;
  const int Npad = a.nT * kTile;
  const long long rows = (long long)a.BH * Npad;
  const unsigned pre_blocks = (unsigned)std::min<long long>((rows + 7) / 8, 148LL * 16);  // one row per warp
  bwd_pre_kernel<256, BF><<<pre_blocks, 256, 0, st>>>(o, dout, lse, a.dq_acc, const_cast<float*>(a.lse2),
                                                       const_cast<float*>(a.Dv), a.N, Npad, rows, a.scale, a.cu_q,
                                                       a.total_q, a.H, a.dl);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  static std::atomic<uint64_t> smem_set{0};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (!(smem_set.load() & (1ull << (dev & 63)))) {
    e = cudaFuncSetAttribute(bwd256_kernel<BF>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    smem_set.fetch_or(1ull << (dev & 63));
  }
  int sms = 0;
  if ((e = device_sm_count(dev, &sms)) != cudaSuccess) return e;
  const long long units = (long long)a.nTk * 2 * a.BH;
  const unsigned grid = (unsigned)std::min<long long>(units, sms);
  if (ev_start && (e = cudaEventRecord(ev_start, st)) != cudaSuccess) return e;
  bwd256_kernel<BF><<<grid, C::kThreads, C::kSmemBytes, st>>>(mq, mk, mv, mdo, mdq, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (ev_stop && (e = cudaEventRecord(ev_stop, st)) != cudaSuccess) return e;
  const long long total_vec8 = (long long)a.BH * (a.cu_q ? Npad : a.N) * a.dl / 8;
  const unsigned blocks = (unsigned)std::min<long long>((total_vec8 + 255) / 256, 148LL * 16);
  bwd_dq_kernel<256, BF><<<blocks, 256, 0, st>>>(a.dq_acc, dq, a.N, Npad, total_vec8, a.cu_q, a.total_q, a.H, a.dl);
  return cudaGetLastError();
}

// Backward of one problem: workspace carve-up, then the head dim's kernels (d <= 64: the 64 kernel, 96 / 128: the 128
// kernel, 256: bwd256_kernel).
inline cudaError_t run_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const CUtensorMap& mdo, const CUtensorMap& mdq, const void* o, const void* dout, const float* lse, void* dq,
                           void* dk, void* dv, int B, int H, int N, int d, float scale, bool causal,
                           const int32_t* key_lens, const int32_t* col_ptr, const int32_t* row_idx, void* workspace,
                           bool bf16, uint64_t budget_ns, cudaStream_t st, cudaEvent_t ev_start,
                           cudaEvent_t ev_stop, const int32_t* cu_q = nullptr, const int32_t* cu_k = nullptr,
                           int total_q = 0, int total_k = 0, int Nk = 0, long long list_head_stride = 0) {
  // packed variable-length batches: N / Nk are the longest query / key sequences; dense: Nk = N
  if (Nk <= 0) Nk = N;
  const int nT = (N + kTile - 1) / kTile;
  const int BH = B * H;
  const size_t npad = (size_t)nT * kTile;
  auto al = [](size_t x) { return (x + 255) / 256 * 256; };
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  BwdArgs a;
  a.dk = dk;
  a.dv = dv;
  a.dq_acc = reinterpret_cast<float*>(ws);
  const size_t side = al((size_t)BH * npad * bwd_row_side_bytes(d));
  a.lse2 = reinterpret_cast<const float*>(ws + al((size_t)BH * npad * d * 4));
  a.Dv = reinterpret_cast<const float*>(ws + al((size_t)BH * npad * d * 4) + side);
  a.dl = d;
  a.key_lens = key_lens;
  a.col_ptr = col_ptr;
  a.row_idx = row_idx;
  a.list_head_stride = list_head_stride;
  a.cu_q = cu_q;
  a.cu_k = cu_k;
  a.total_q = total_q;
  a.total_k = total_k;
  a.H = H;
  a.N = N;
  a.nT = nT;
  a.Nk = Nk;
  a.nTk = (Nk + kTile - 1) / kTile;
  a.BH = BH;
  a.causal = causal ? 1 : 0;
  a.scale = scale;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.budget_ns = budget_ns;
  if (d == 256)
    return bf16 ? launch_bwd256<true>(mq, mk, mv, mdo, mdq, o, dout, lse, dq, a, st, ev_start, ev_stop)
                : launch_bwd256<false>(mq, mk, mv, mdo, mdq, o, dout, lse, dq, a, st, ev_start, ev_stop);
  if (d <= 64)  // 32 runs on the 64 kernel
    return bf16 ? launch_bwd<64, true>(mq, mk, mv, mdo, mdq, o, dout, lse, dq, a, st, ev_start, ev_stop)
                : launch_bwd<64, false>(mq, mk, mv, mdo, mdq, o, dout, lse, dq, a, st, ev_start, ev_stop);
  return bf16 ? launch_bwd<128, true>(mq, mk, mv, mdo, mdq, o, dout, lse, dq, a, st, ev_start, ev_stop)
              : launch_bwd<128, false>(mq, mk, mv, mdo, mdq, o, dout, lse, dq, a, st, ev_start, ev_stop);
}

}  // namespace fa
