// fa_fwd256.cuh -- forward kernel for head dimension 256 on sm_100a.
//
// Same method as fa_fwd.cuh (FlashAttention review page, "Method"; explainer page, "online softmax"): K/V tiles
// stream past a resident 128-row Q tile, the running max and denominator stay on chip, O and the per-row
// logsumexp are the only outputs.  What changes at d = 256 is the fit on the SM:
//   * TMEM (512 columns) holds one Q tile's O (256 columns) and TWO score buffers S_0, S_1 (128 columns each),
//     so the score MMA of K/V tile j+2 is issued as soon as P_j V_j is and runs while the softmax warps work on
//     tile j+1: within one Q tile the softmax and the tensor core overlap, and S is normally complete before the
//     softmax warps get to it.  (At d <= 128 two Q tiles ping-pong instead; here two O accumulators would not fit.)
//   * Shared memory holds Q (64 KB) and a ring of ten 16 KB chunks: a K tile arrives as four chunks of 64 head
//     dims (128 keys each, the K-dimension of Q K^T), a V tile as four chunks of 32 keys (all 256 dims, the
//     K-dimension of P V, read as an N = 256 operand).  The TMA warp fetches K two tiles ahead of V (K_0, K_1,
//     V_0, K_2, V_1, ...), the order in which the MMA thread consumes them (see the issue order below).
//
// Roles (192 threads, one CTA per SM, persistent over 128-row Q tiles ordered longest first):
//   warps 0-3  softmax and epilogue: thread = query row = TMEM lane, whole rows, no shuffles;
//   warp 4     MMA issuer (one thread): S_b = Q K_j^T (b = step parity), O += P_b V_j (P_b from TMEM);
//   warp 5     TMA producer.
// Barrier phases and ring positions run on across the CTA's units, as in fa_fwd.cuh.
#pragma once
#include "fa_fwd.cuh"

namespace fa {

struct Fwd256Cfg {
  static constexpr int D = 256;
  static constexpr int kChunkBytes = 16384;  // 128 keys x 64 dims (K) or 32 keys x 256 dims (V), 16-bit
  static constexpr int kChunks = 4;          // chunks per K or V tile
  static constexpr int kNumSlots = 10;
  static constexpr int kQBytes = kTile * D * 2;
  static constexpr int kSmemBytes = kQBytes + kNumSlots * kChunkBytes + 1024;
  static constexpr int kWarpMma = 4, kWarpLoad = 5;
  static constexpr int kThreads = 192;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;  // S_0 [0,128), S_1 [128,256), O [256,512)
};

// The CTA's stream of (unit, visible K/V tile) steps: units in UnitSeq order, tiles in list order, units with no
// visible tile skipped.  The TMA and MMA roles run these ahead of the per-unit loop of the softmax warps.
template <int kMode>
struct StepWalker {
  UnitSeq us;
  PairTileIter it;
  FwdUnit u;
  bool live;
  __device__ __forceinline__ void init(int total_units) {
    us.init(total_units);
    live = false;
  }
  // Next step: its K/V tile j; `fresh` when the step is the first of its unit.  False once the stream is over.
  __device__ __forceinline__ bool next(const FwdArgs& a, int& j, bool& fresh) {
    fresh = false;
    int fl;
    while (true) {
      if (live && it.next(j, fl)) return true;
      int L;
      if (!us.next(L)) {
        live = false;
        return false;
      }
      u = fwd_unit<kMode>(L, a, 1);
      fwd_tiles(it, u, a);
      live = true;
      fresh = true;
    }
  }
};

// The same stream one step ahead: the caller can see whether the next step opens a unit (ok_nx, fresh_nx) and
// whether the step it takes closes one (`last`).  u is the unit of the step last returned.
template <int kMode>
struct LookaheadWalker {
  StepWalker<kMode> w;
  FwdUnit u, u_nx;
  bool ok_nx, fresh_nx;
  int j_nx;
  __device__ __forceinline__ void init(int total_units, const FwdArgs& a) {
    w.init(total_units);
    ok_nx = w.next(a, j_nx, fresh_nx);
    u_nx = w.u;
  }
  __device__ __forceinline__ bool next(const FwdArgs& a, int& j, bool& fresh, bool& last) {
    if (!ok_nx) return false;
    j = j_nx;
    fresh = fresh_nx;
    u = u_nx;
    ok_nx = w.next(a, j_nx, fresh_nx);
    u_nx = w.u;
    last = !ok_nx || fresh_nx;
    return true;
  }
};

// Issue order shared by the TMA and MMA roles (ring chunks are consumed in the order they are produced):
//   S (or K) runs two steps ahead of P V (or V): after P_j V_j comes S_{j+2};
//   except that a unit's first S waits until every P V of the previous unit has been issued -- it waits for the
//   new Q, and the previous unit's last P V (and so its epilogue) must not wait behind that.
// So across a unit boundary the order is ..., P V_{n-2}, P V_{n-1}, S_n, S_{n+1}, P V_n, S_{n+2}, ...
// The Q buffer is released right after a unit's last S, one step before the next unit's first S is due.

template <bool kBF16, int kMode>
__global__ void __launch_bounds__(Fwd256Cfg::kThreads, 1)
    fwd256_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v, const FwdArgs args) {
  using C = Fwd256Cfg;
  constexpr int D = C::D;
  constexpr int NS = C::kNumSlots;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sR = smem + C::kQBytes;

  __shared__ __align__(8) uint64_t bar_q, bar_q_free, bar_full[NS], bar_empty[NS], bar_s[2], bar_p[2], bar_pv,
      bar_o, bar_o_free, bar_drain;
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
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(ptx::smem_addr(&bar_full[s]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(ptx::smem_addr(&bar_s[b]), 1);
      ptx::mbar_init(ptx::smem_addr(&bar_p[b]), 128);
    }
    ptx::mbar_init(ptx::smem_addr(&bar_pv), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_o), 1);
    ptx::mbar_init(ptx::smem_addr(&bar_o_free), 128);
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

  if (warp == C::kWarpLoad) {
    // ------------------------------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      ptx::prefetch_tensormap(&map_q);
      ptx::prefetch_tensormap(&map_k);
      ptx::prefetch_tensormap(&map_v);
      const uint32_t bq = ptx::smem_addr(&bar_q);
      LookaheadWalker<kMode> kw;
      StepWalker<kMode> vw;
      kw.init(total_units, args);
      vw.init(total_units);
      int n = 0, nq = 0;  // ring chunks issued, Q tiles issued
      int kc = 0, vc = 0;  // K tiles and V tiles issued
      bool ok = true;
      // next free ring slot (waits for its previous chunk to be consumed); arms its full barrier
      auto slot = [&](uint32_t& dst, uint32_t& bf) -> bool {
        const int s = n % NS;
        const uint32_t ph = (n / NS) & 1;
        if (!wait_or_abort(ptx::smem_addr(&bar_empty[s]), ph ^ 1, args.budget_ns, abortp)) return false;
        dst = ptx::smem_addr(sR + s * C::kChunkBytes);
        bf = ptx::smem_addr(&bar_full[s]);
        ptx::mbar_arrive_expect_tx(bf, C::kChunkBytes);
        ++n;
        return true;
      };
      // K of the next step (and that unit's Q first when the step opens a unit)
      auto load_k = [&]() -> bool {
        int j;
        bool fresh, last;
        if (!kw.next(args, j, fresh, last)) return true;
        ++kc;
        const FwdUnit& u = kw.u;
        if (fresh) {
          // the Q buffer is free once every S MMA of the previous unit has completed
          if (nq > 0 && !wait_or_abort(ptx::smem_addr(&bar_q_free), (nq - 1) & 1, args.budget_ns, abortp))
            return false;
          ptx::mbar_arrive_expect_tx(bq, C::kQBytes);
          for (int c = 0; c < D / 64; ++c)
            tma_rows(ptx::smem_addr(sQ + c * 16384), &map_q, c, u.qt0 * kTile, u.g.q0, u.bh, u.h, packed, bq);
          ++nq;
        }
        for (int c = 0; c < C::kChunks; ++c) {  // chunk c: head dims [64c, 64c+64) of 128 keys
          uint32_t dst, bf;
          if (!slot(dst, bf)) return false;
          tma_rows(dst, &map_k, c, j * kTile, u.g.k0, u.bh, u.h, packed, bf);
        }
        return true;
      };
      // K tiles up to two steps ahead of V; a unit's first K only once every V before it is issued
      auto top_up = [&]() -> bool {
        while (kc < vc + 2 && kw.ok_nx) {
          if (kw.fresh_nx && kc != vc) break;
          if (!load_k()) return false;
        }
        return true;
      };
      ok = top_up();
      while (ok) {
        int j;
        bool fresh;
        if (!vw.next(args, j, fresh)) break;
        const FwdUnit& u = vw.u;
        for (int c = 0; c < C::kChunks && ok; ++c) {  // chunk c: keys [32c, 32c+32), four 64-dim boxes
          uint32_t dst, bf;
          if (!(ok = slot(dst, bf))) break;
          for (int cb = 0; cb < D / 64; ++cb)
            tma_rows(dst + cb * 4096, &map_v, cb, j * kTile + 32 * c, u.g.k0, u.bh, u.h, packed, bf);
        }
        ++vc;
        if (ok) ok = top_up();
      }
      // Let every copy this thread issued land before the CTA can exit (immediate in the normal path).
      if (nq > 0) ptx::mbar_wait(bq, (nq - 1) & 1, args.budget_ns);
      for (int k = (n > NS ? n - NS : 0); k < n; ++k)
        ptx::mbar_wait(ptx::smem_addr(&bar_full[k % NS]), (k / NS) & 1, args.budget_ns);
    }
  } else if (warp == C::kWarpMma) {
    // ------------------------------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = ptx::idesc_f16(kBF16, false, false, 128, 128);
      constexpr uint32_t idesc_o = ptx::idesc_f16(kBF16, false, true, 128, D);
      const uint64_t dq0 = ptx::sw128_desc(ptx::smem_addr(sQ), 16, 1024);   // Q: 4 blocks of 64 dims, K-major
      const uint64_t dk0 = ptx::sw128_desc(ptx::smem_addr(sR), 16, 1024);   // K chunk, K-major
      const uint64_t dv0 = ptx::sw128_desc(ptx::smem_addr(sR), 4096, 1024); // V chunk, N-major, 4 KB per 64 dims
      int n = 0;           // ring chunks consumed (same order as issued by the TMA warp)
      int gs = 0, nq = 0;  // S steps issued, Q tiles used
      bool ok = true;
      // the next kChunks ring chunks (one K or V tile), all waited for before any of their MMAs is issued: on
      // sm_100a each wait of the issuing thread lets its queued MMAs drain first
      auto chunks = [&](int (&slots)[C::kChunks]) -> bool {
        for (int c = 0; c < C::kChunks; ++c) {
          slots[c] = n % NS;
          const uint32_t ph = (n / NS) & 1;
          ++n;
          if (!wait_or_abort(ptx::smem_addr(&bar_full[slots[c]]), ph, args.budget_ns, abortp)) return false;
        }
        ptx::tc_fence_after();
        return true;
      };
      LookaheadWalker<kMode> sw;
      sw.init(total_units, args);
      // S_b = Q K_j^T for the next step of the stream (b = its parity); nothing when the stream is over
      auto issue_next_s = [&]() -> bool {
        int j;
        bool fresh, last;
        if (!sw.next(args, j, fresh, last)) return true;
        if (fresh) {
          if (!wait_or_abort(ptx::smem_addr(&bar_q), nq & 1, args.budget_ns, abortp)) return false;
          ptx::tc_fence_after();
          ++nq;
        }
        const uint32_t d_s = tmem + (gs & 1) * 128;
        int slots[C::kChunks];
        if (!chunks(slots)) return false;
        for (int c = 0; c < C::kChunks; ++c) {
          const int s = slots[c];
          const uint64_t a = ptx::desc_advance(dq0, c * 16384);
          const uint64_t b = ptx::desc_advance(dk0, s * C::kChunkBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            ptx::mma_ss(d_s, ptx::desc_advance(a, kk * 32), ptx::desc_advance(b, kk * 32), idesc_s,
                        (c > 0 || kk > 0) ? 1u : 0u);
          ptx::mma_commit(ptx::smem_addr(&bar_empty[s]));
        }
        ptx::mma_commit(ptx::smem_addr(&bar_s[gs & 1]));
        if (last) ptx::mma_commit(ptx::smem_addr(&bar_q_free));  // every S of this unit issued
        ++gs;
        return true;
      };
      int gp = 0, ku = 0;  // P V steps issued, units finished
      // S up to two steps ahead of P V; a unit's first S only at a unit end (allow_fresh) with every P V issued
      auto top_up = [&](bool allow_fresh) -> bool {
        while (gs < gp + 2 && sw.ok_nx) {
          if (sw.fresh_nx && !(allow_fresh && gs == gp)) break;
          if (!issue_next_s()) return false;
        }
        return true;
      };
      ok = top_up(true);
      UnitSeq us;
      us.init(total_units);
      int L;
      while (ok && us.next(L)) {
        const FwdUnit u = fwd_unit<kMode>(L, args, 1);
        PairTileIter it;
        fwd_tiles(it, u, args);
        int li = 0, j, fl;
        while (ok && it.next(j, fl)) {
          if (!(ok = wait_or_abort(ptx::smem_addr(&bar_p[gp & 1]), (gp >> 1) & 1, args.budget_ns, abortp))) break;
          // the first P V of a unit overwrites O: the epilogue must have read the previous unit's
          if (li == 0 && ku > 0 &&
              !(ok = wait_or_abort(ptx::smem_addr(&bar_o_free), (ku - 1) & 1, args.budget_ns, abortp)))
            break;
          ptx::tc_fence_after();
          const uint32_t p_col = tmem + (gp & 1) * 128;
          int slots[C::kChunks];
          if (!(ok = chunks(slots))) break;
          for (int kc = 0; kc < C::kChunks; ++kc) {
            const int s = slots[kc];
            const uint64_t b = ptx::desc_advance(dv0, s * C::kChunkBytes);
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2)  // 16 keys each; P packs two keys per column
              ptx::mma_ts(tmem + C::kColO, p_col + (2 * kc + k2) * 8, ptx::desc_advance(b, k2 * 2048), idesc_o,
                          (li > 0 || kc > 0 || k2 > 0) ? 1u : 0u);
            ptx::mma_commit(ptx::smem_addr(&bar_empty[s]));
          }
          if (!ok) break;
          ptx::mma_commit(ptx::smem_addr(&bar_pv));
          ++gp;
          ++li;
          ok = top_up(false);  // S two steps ahead; its buffer's P was read by the P V just issued
        }
        if (!ok) break;
        // a unit with no P V waits for the previous epilogue here, so bar_o never runs two phases ahead
        if (li == 0 && ku > 0 &&
            !(ok = wait_or_abort(ptx::smem_addr(&bar_o_free), (ku - 1) & 1, args.budget_ns, abortp)))
          break;
        ptx::mma_commit(ptx::smem_addr(&bar_o));
        ++ku;
        ok = top_up(true);  // the next unit's first S (and the one after)
      }
      // No MMA may still be running when the tensor memory is released.
      ptx::mma_commit(ptx::smem_addr(&bar_drain));
      ptx::mbar_wait(ptx::smem_addr(&bar_drain), 0, args.budget_ns);
    }
  } else {
    // ------------------------------------------------------------------------------------------ softmax warps
    const int quarter = warp;
    const int row = quarter * 32 + lane;  // row within the Q tile == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_base + C::kColO;
    const float scale_log2 = args.scale_log2;
    int g = 0, ku = 0;  // steps (global across units), units
    bool ok = true;
    UnitSeq us;
    us.init(total_units);
    int L;
    while (ok && us.next(L)) {
      FwdUnit u = fwd_unit<kMode>(L, args, 1);
      PairTileIter it;
      fwd_tiles(it, u, args);
      const int qt = u.qt0;
      const int grow = qt * kTile + row;  // row within the sequence
      const int kv_lim = u.kv_lim;
      int coff = 0;  // split-K/V causal: keys c <= grow + coff
      if constexpr (split) coff = u.off;
      float m_ref = -INFINITY;
      ptx::f32x2 lacc[2] = {{0.f, 0.f}, {0.f, 0.f}};
      int kidx = 0, j, fl;
      while (it.next(j, fl)) {
        const int b = g & 1;
        ok = __all_sync(0xffffffffu,
                        wait_or_abort(ptx::smem_addr(&bar_s[b]), (g >> 1) & 1, args.budget_ns, abortp));
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t tS = tmem + lane_base + b * 128;
        uint32_t sr[128];
        ptx::tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        ptx::tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        ptx::tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        ptx::tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        ptx::tmem_ld_wait();
        float* s = reinterpret_cast<float*>(sr);
        if constexpr (split) {
          if ((causal && (j + 1) * kTile - 1 > qt * kTile + coff) || (j + 1) * kTile > kv_lim) {
            const int c0 = j * kTile;
            const int lim = causal ? min(kv_lim, grow + 1 + coff) : kv_lim;
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (c0 + i >= lim) s[i] = -INFINITY;
          }
        } else {
          if ((causal && j >= qt) || (j + 1) * kTile > kv_lim) {
            const int c0 = j * kTile;
            const int lim = causal ? min(kv_lim, grow + 1) : kv_lim;
#pragma unroll
            for (int i = 0; i < 128; ++i)
              if (c0 + i >= lim) s[i] = -INFINITY;
          }
        }
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
        const bool need = m_tile > m_ref + 8.0f;  // lazy rescale, as in fa_fwd.cuh
        float alpha = 1.0f;
        if (need) {
          alpha = ptx::ex2(m_ref - m_tile);
          m_ref = m_tile;
        }
        const float m_use = (m_ref == -INFINITY) ? 0.0f : m_ref;
        if (need) {
          lacc[0].x *= alpha; lacc[0].y *= alpha; lacc[1].x *= alpha; lacc[1].y *= alpha;
        }
        const ptx::f32x2 sc2{scale_log2, scale_log2}, nm2{-m_use, -m_use};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const ptx::f32x2 x = ptx::fma2({s[h * 64 + 2 * i], s[h * 64 + 2 * i + 1]}, sc2, nm2);
            const bool emu = kExpFmaEvery > 0 && (i % (kExpFmaEvery > 0 ? kExpFmaEvery : 1)) == kExpFmaEvery - 1;
            const float p0 = emu ? ptx::exp2_fma(x.x) : ptx::ex2(x.x);
            const float p1 = emu ? ptx::exp2_fma(x.y) : ptx::ex2(x.y);
            pk[i] = ptx::pack2<kBF16>(p0, p1);
            lacc[i & 1] = ptx::add2(lacc[i & 1], ptx::unpack2<kBF16>(pk[i]));
          }
          ptx::tmem_st32(tS + h * 32, pk);
        }
        if (kidx > 0) {
          // P V of the previous step must be complete before O is touched.  Waited every step (it is normally
          // long done) so the phase of bar_pv is never more than one behind.
          ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_pv), (g - 1) & 1, args.budget_ns, abortp));
          if (!ok) break;
          if (__any_sync(0xffffffffu, need)) {
            ptx::tc_fence_after();
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
        }
        ptx::tmem_st_wait();
        ptx::tc_fence_before();
        ptx::mbar_arrive(ptx::smem_addr(&bar_p[b]));
        ++g;
        ++kidx;
      }
      if (!ok) break;
      // ---------------------------------------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, wait_or_abort(ptx::smem_addr(&bar_o), ku & 1, args.budget_ns, abortp));
      if (!ok) break;
      ptx::tc_fence_after();
      const bool row_ok = grow < u.g.lq;
      const float l_sum = (lacc[0].x + lacc[0].y) + (lacc[1].x + lacc[1].y);
      const bool nonempty = l_sum > 0.f;
      const float inv = nonempty ? 1.0f / l_sum : 0.0f;
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
          ptx::mbar_arrive(ptx::smem_addr(&bar_o_free));
        }
        if constexpr (split) {
          if (row_ok && in_bounds(prow < part_rows, kSiteFwd256)) {
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
          if (row_ok && in_bounds(orow_idx < o_rows, kSiteFwd256)) {
            uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
            for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
        }
      }
      if (row_ok) {
        const float lse_v = nonempty ? (m_ref + __log2f(l_sum)) * 0.69314718055994530942f : -INFINITY;
        if constexpr (split) {
          if (in_bounds(prow < part_rows, kSiteFwd256)) args.lse_part[prow] = lse_v;
        } else {
          const size_t li = packed ? (size_t)u.h * args.total_q + u.g.q0 + grow : (size_t)u.bh * args.N + grow;
          if (in_bounds(li < o_rows, kSiteFwd256)) args.lse[li] = lse_v;
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

}  // namespace fa
