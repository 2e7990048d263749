// Flash-style attention on tcgen05/TMEM, in three modes that share one pipeline:
//
//   kDense    : O = softmax(scale Q K^T) V over all N keys, plus the per-query log-sum-exp
//               (the anchor's dense attention and the first of the two selection passes).
//   kReuse    : group g's C queries (rows perm[g*C ...]) attend to the k keys idx[g, :],
//               renormalised over that set, then the cached residual R is added:
//               O_hat = SparseAttn(Q, K, V; G, S) + R.
//   kResidual : same sparse attention on the anchor's own inputs; writes R = O_full - O_s.
//
// The method: "MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", sections 무엇과 다른가
// (anchor/reuse alternation, O_hat = SparseAttn(...) + R with R = O_full - O_sparse) and
// 어떻게 쓰나 (the kernel gathers individual K/V tokens online from the cached indices; query
// groups are exactly one query tile).
//
// One CTA per SM, persistent over work units (one 128-row query tile each).  Warp roles:
//   warps 0-3  softmax + epilogue: thread t owns tile row t = TMEM lane t;
//   warps 4-7  producer: cp.async gathers of Q rows (by perm) and K/V rows (by idx) into
//              128-byte-swizzled K-major tiles, a STAGES-deep ring for K/V; the 128 indices
//              of a tile are fetched one tile ahead with one coalesced load per thread and
//              staged in shared memory, so no copy waits on an index load;
//   warp 8     TMEM allocator and the single MMA-issuing thread.
// TMEM (512 columns): S = Q K^T in two 128-column buffers, O (d columns), and P in two
// 64-column buffers (bf16 pairs).  Softmax reads S, writes P back to TMEM; O += P V runs with
// A = P from TMEM and B = V (an MN-major shared-memory operand).  The running max is raised
// lazily (only when it grows by more than 2^8), so O is rescaled in TMEM rarely.
#pragma once

#include "sm100.cuh"

namespace mcs {

enum AttnMode : int { kDense = 0, kReuse = 1, kResidual = 2 };

struct AttnParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  const int32_t* perm;           // [BH, N]   sparse modes
  const int32_t* idx;            // [BH, G, k] sparse modes
  const __nv_bfloat16* R_in;     // kReuse: residual to add (nullable)
  const __nv_bfloat16* O_full;   // kResidual: dense output of the anchor
  __nv_bfloat16* out;            // kDense: O; kReuse: O_hat; kResidual: R
  float* lse;                    // kDense: natural-log LSE [BH, N] (nullable)
  int BH, N, C, G, k;
  int units_per_head;            // dense: ceil(N/128); sparse: G
  int kv_tiles;                  // dense: ceil(N/128); sparse: ceil(k/128)
  int kv_count;                  // dense: N; sparse: k
  int num_units;                 // BH * units_per_head
  float scale_log2;              // scale * log2(e)
  int store_out;                 // kDense: 0 = LSE only
};

constexpr int kAttnThreads = 288;
constexpr int kTile = 128;

template <int HD>
struct AttnSmem {
  static constexpr uint32_t TILE_BYTES = kTile * HD * 2;  // Q, K or V tile
  static constexpr int STAGES = HD == 128 ? 3 : 6;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + TILE_BYTES;
  static constexpr uint32_t V_OFF = K_OFF + STAGES * TILE_BYTES;
  static constexpr uint32_t IDX_OFF = V_OFF + STAGES * TILE_BYTES;  // 2 x 128 KV indices
  static constexpr uint32_t QIDX_OFF = IDX_OFF + 2 * kTile * 4;     // 128 query indices
  static constexpr uint32_t BAR_OFF = QIDX_OFF + kTile * 4;
  // barriers: q_full, q_empty, k_full[S], v_full[S], kv_empty[S], s_full[2], s_empty[2],
  //           p_full, pv_done[2], o_empty, drain
  static constexpr int NBAR = 2 + 3 * STAGES + 4 + 1 + 2 + 2;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr uint32_t BYTES = MISC_OFF + 16 + 1024;  // + alignment slack
  static_assert(BYTES <= 232448, "shared memory budget");
};

// TMEM column map (512 columns allocated)
constexpr uint32_t kTmS = 0;      // two S buffers, 128 columns each
constexpr uint32_t kTmO = 256;    // O, d columns
constexpr uint32_t kTmP = 384;    // two P buffers, 64 columns each

template <int HD, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_kernel(const AttnParams p) {
  using L = AttnSmem<HD>;
  constexpr int STAGES = L::STAGES;
  constexpr int CHUNKS = HD / 8;                      // 16-byte chunks per row
  constexpr uint32_t HALF = kTile * 128;               // bytes per 64-column half of a tile
  constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, HD, false, true);
  constexpr bool SPARSE = MODE != kDense;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* gptr = smem_raw + (base - raw_addr);

  uint64_t* bars = reinterpret_cast<uint64_t*>(gptr + L::BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* v_full = k_full + STAGES;
  uint64_t* kv_empty = v_full + STAGES;
  uint64_t* s_full = kv_empty + STAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_done = p_full + 1;   // [2], by tile parity
  uint64_t* o_empty = pv_done + 2;
  uint64_t* drain = o_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gptr + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gptr + L::MISC_OFF + 4);
  int32_t* sIdx = reinterpret_cast<int32_t*>(gptr + L::IDX_OFF);
  int32_t* sQidx = reinterpret_cast<int32_t*>(gptr + L::QIDX_OFF);

  const uint32_t sQ = base + L::Q_OFF;
  const uint32_t sK = base + L::K_OFF;
  const uint32_t sV = base + L::V_OFF;
  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    mbar_init(q_empty, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(k_full + s, 128);
      mbar_init(v_full + s, 128);
      mbar_init(kv_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, 128);
      mbar_init(pv_done + b, 1);
    }
    mbar_init(p_full, 128);
    mbar_init(o_empty, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int T = p.kv_tiles;

  if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ producer
    const int pt = threadIdx.x - 128;
    uint32_t kv_it = 0, u_it = 0;
    for (int unit = blockIdx.x; unit < p.num_units; unit += gridDim.x, ++u_it) {
      const int bh = unit / p.units_per_head;
      const int ut = unit - bh * p.units_per_head;
      const size_t head_off = static_cast<size_t>(bh) * p.N;
      const int32_t* idx_row = SPARSE ? p.idx + (static_cast<size_t>(bh) * p.G + ut) * p.k : nullptr;
      // index loads for this unit's Q tile and first KV tile, issued before any wait
      int qi = -1, nidx = -1;
      if (SPARSE) {
        if (pt < p.C) qi = p.perm[head_off + static_cast<size_t>(ut) * p.C + pt];
        if (pt < p.kv_count) nidx = idx_row[pt];
      }
      if (!mbar_wait(q_empty, (u_it & 1) ^ 1, abort_flag)) break;
      if (SPARSE) {
        if (qi != -1 && static_cast<unsigned>(qi) >= static_cast<unsigned>(p.N)) {
          raise_status(kStatusBadIndex);
          qi = -1;
        }
        sQidx[pt] = qi;
        named_sync(2, 128);
      }
#pragma unroll 4
      for (int it = 0; it < CHUNKS; ++it) {
        const int lin = it * 128 + pt;
        const int r = lin / CHUNKS, c = lin % CHUNKS;
        int q;
        bool ok;
        if (SPARSE) {
          q = sQidx[r];
          ok = q >= 0;
        } else {
          q = ut * kTile + r;
          ok = q < p.N;
        }
        const __nv_bfloat16* src = p.Q + ((head_off + (ok ? q : 0)) * HD + c * 8);
        cp_async16(sQ + sw128_offset(r, c, kTile), src, ok ? 16u : 0u);
      }
      cp_async_arrive(q_full);
      for (int j = 0; j < T; ++j, ++kv_it) {
        const uint32_t st = kv_it % STAGES;
        int32_t* tidx = sIdx + (j & 1) * kTile;
        if (SPARSE) {
          int cur = nidx;
          if (cur != -1 && static_cast<unsigned>(cur) >= static_cast<unsigned>(p.N)) {
            raise_status(kStatusBadIndex);
            cur = -1;
          }
          tidx[pt] = cur;
          const int pos = (j + 1) * kTile + pt;
          nidx = (j + 1 < T && pos < p.kv_count) ? idx_row[pos] : -1;  // prefetch the next tile
        }
        if (!mbar_wait(kv_empty + st, ((kv_it / STAGES) & 1) ^ 1, abort_flag)) break;
        if (SPARSE) named_sync(2, 128);
        const uint32_t dK = sK + st * L::TILE_BYTES, dV = sV + st * L::TILE_BYTES;
        // K rows, then V rows, each followed by its own arrival so QK^T can start early.
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
          const __nv_bfloat16* gsrc = which == 0 ? p.K : p.V;
          const uint32_t dst = which == 0 ? dK : dV;
#pragma unroll 4
          for (int it = 0; it < CHUNKS; ++it) {
            const int lin = it * 128 + pt;
            const int r = lin / CHUNKS, c = lin % CHUNKS;
            int kv;
            bool ok;
            if (SPARSE) {
              kv = tidx[r];
              ok = kv >= 0;
            } else {
              kv = j * kTile + r;
              ok = kv < p.kv_count;
            }
            const __nv_bfloat16* src = gsrc + ((head_off + (ok ? kv : 0)) * HD + c * 8);
            cp_async16(dst + sw128_offset(r, c, kTile), src, ok ? 16u : 0u);
          }
          cp_async_arrive(which == 0 ? k_full + st : v_full + st);
        }
      }
      if (*abort_flag) break;
    }
    cp_async_wait_all();
  } else if (warp == 8) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS = tmem + kTmS, tO = tmem + kTmO, tP = tmem + kTmP;
      uint32_t kv_base = 0, s_base = 0, u_it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x, ++u_it) {
        ok = mbar_wait(q_full, u_it & 1, abort_flag);
        if (!ok) break;
        auto issue_qk = [&](int j) -> bool {
          const uint32_t it = kv_base + j, st = it % STAGES;
          if (!mbar_wait(k_full + st, (it / STAGES) & 1, abort_flag)) return false;
          const uint32_t si = s_base + j, b = si & 1;
          if (!mbar_wait(s_empty + b, ((si >> 1) & 1) ^ 1, abort_flag)) return false;
          fence_proxy_async_smem();
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks) {
            const uint32_t koff = (ks >> 2) * HALF + (ks & 3) * 32;
            const uint64_t ad = desc_sw128(sQ + koff, 16, 1024);
            const uint64_t bd = desc_sw128(sK + st * L::TILE_BYTES + koff, 16, 1024);
            mma_bf16_ss(tS + b * 128, ad, bd, IDESC_QK, ks > 0 ? 1u : 0u);
          }
          mma_commit(s_full + b);
          return true;
        };
        auto issue_pv = [&](int j) -> bool {
          const uint32_t it = kv_base + j, st = it % STAGES;
          const uint32_t si = s_base + j, b = si & 1;
          if (!mbar_wait(p_full, si & 1, abort_flag)) return false;
          if (!mbar_wait(v_full + st, (it / STAGES) & 1, abort_flag)) return false;
          if (j == 0 && !mbar_wait(o_empty, (u_it & 1) ^ 1, abort_flag)) return false;
          fence_proxy_async_smem();
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks) {
            const uint64_t bd = desc_sw128(sV + st * L::TILE_BYTES + ks * 2048, HALF, 1024);
            mma_bf16_ts(tO, tP + b * 64 + ks * 8, bd, IDESC_PV, (j > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(kv_empty + st);
          mma_commit(pv_done + b);
          return true;
        };
        ok = issue_qk(0);
        if (ok && T > 1) ok = issue_qk(1);
        if (ok && T <= 2) mma_commit(q_empty);
        for (int j = 0; j < T && ok; ++j) {
          ok = issue_pv(j);
          if (ok && j + 2 < T) {
            ok = issue_qk(j + 2);
            if (ok && j + 3 == T) mma_commit(q_empty);
          }
        }
        kv_base += T;
        s_base += T;
      }
      // drain: every MMA issued above has completed before TMEM is released
      mma_commit(drain);
      uint64_t t0 = globaltimer_ns();
      while (!mbar_test(drain, 0)) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
          raise_status(kStatusTimeout);
          break;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int row = threadIdx.x;  // 0..127 == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base + kTmS, tO = tmem + lane_base + kTmO, tP = tmem + lane_base + kTmP;
    const float sl2 = p.scale_log2;
    uint32_t s_base = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x) {
      const int bh = unit / p.units_per_head;
      const int ut = unit - bh * p.units_per_head;
      float m_used = -INFINITY, l_sum = 0.f;
      for (int j = 0; j < T; ++j) {
        const uint32_t si = s_base + j, b = si & 1;
        if (!mbar_wait_warp(s_full + b, (si >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(tS + b * 128 + 0, sr);
        tmem_ld32(tS + b * 128 + 32, sr + 32);
        tmem_ld32(tS + b * 128 + 64, sr + 64);
        tmem_ld32(tS + b * 128 + 96, sr + 96);
        tmem_ld_wait_regs(sr);
        reg_fence32(sr + 32);
        reg_fence32(sr + 64);
        reg_fence32(sr + 96);
        tc_fence_before();
        mbar_arrive(s_empty + b);
        const int valid = min(kTile, p.kv_count - j * kTile);
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 128; ++c) {
          const float v = c < valid ? __uint_as_float(sr[c]) : -INFINITY;
          mx = fmaxf(mx, v);
        }
        const float m_tile = mx * sl2;
        float m_new = m_used, alpha = 1.f;
        const bool raise = m_tile > m_used + 8.f;
        if (raise) {
          m_new = m_tile;
          alpha = fast_exp2(m_used - m_new);  // 0 on the first tile
        }
        // P buffer b was last read by PV of tile si-2
        if (!mbar_wait_warp(pv_done + b, ((si >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        float rs = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t pw[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = q * 32 + 2 * i;
            const float e0 = c < valid ? fast_exp2(fmaf(__uint_as_float(sr[c]), sl2, -m_new)) : 0.f;
            const float e1 = c + 1 < valid ? fast_exp2(fmaf(__uint_as_float(sr[c + 1]), sl2, -m_new)) : 0.f;
            rs += e0 + e1;
            pw[i] = pack_bf16x2(e0, e1);
          }
          tmem_st16(tP + b * 64 + q * 16, pw);
        }
        l_sum = l_sum * alpha + rs;
        m_used = m_new;
        // tcgen05.ld/st are warp-collective: rescale the warp's rows if any of them needs it
        // (alpha is 1 for rows whose max did not move); O must hold PV of tile si-1 first
        if (j > 0 && __any_sync(0xffffffffu, raise)) {
          if (!mbar_wait_warp(pv_done + (b ^ 1), ((si - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c0 = 0; c0 < HD; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c0, o);
            tmem_ld_wait_regs(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c0, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok) break;
      const uint32_t si_last = s_base + T - 1;
      if (!mbar_wait_warp(pv_done + (si_last & 1), (si_last >> 1) & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // ---- epilogue: this thread's output row
      int q;
      bool live;
      if (SPARSE) {
        live = row < p.C;
        q = live ? p.perm[static_cast<size_t>(bh) * p.N + static_cast<size_t>(ut) * p.C + row] : 0;
        if (live && static_cast<unsigned>(q) >= static_cast<unsigned>(p.N)) live = false;
      } else {
        q = ut * kTile + row;
        live = q < p.N;
      }
      const float inv_l = 1.f / l_sum;
      const size_t rbase = (static_cast<size_t>(bh) * p.N + q) * HD;
#pragma unroll 1
      for (int c0 = 0; c0 < HD; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(tO + c0, o);
        tmem_ld_wait_regs(o);
        if (live && (MODE != kDense || p.store_out)) {
#pragma unroll
          for (int c = 0; c < 32; c += 8) {
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(o[c + i]) * inv_l;
            if (MODE == kReuse && p.R_in != nullptr) {
              const uint4 rr = *reinterpret_cast<const uint4*>(p.R_in + rbase + c0 + c);
              const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rr);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(r2[i]);
                v[2 * i] += f.x;
                v[2 * i + 1] += f.y;
              }
            } else if (MODE == kResidual) {
              const uint4 rr = *reinterpret_cast<const uint4*>(p.O_full + rbase + c0 + c);
              const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rr);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(r2[i]);
                v[2 * i] = f.x - v[2 * i];
                v[2 * i + 1] = f.y - v[2 * i + 1];
              }
            }
            uint4 w;
            w.x = pack_bf16x2(v[0], v[1]);
            w.y = pack_bf16x2(v[2], v[3]);
            w.z = pack_bf16x2(v[4], v[5]);
            w.w = pack_bf16x2(v[6], v[7]);
            *reinterpret_cast<uint4*>(p.out + rbase + c0 + c) = w;
          }
        }
      }
      if (MODE == kDense && live && p.lse != nullptr) {
        p.lse[static_cast<size_t>(bh) * p.N + q] = (m_used + __log2f(l_sum)) * 0.69314718055994531f;
      }
      tc_fence_before();
      mbar_arrive(o_empty);
      s_base += T;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mcs
