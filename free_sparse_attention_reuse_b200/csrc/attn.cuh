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
//   warps 0-7  softmax + epilogue: warp w owns tile rows 32*(w%4) .. +31 (its TMEM lanes) and
//              the column half w/4 of S, P and O; each warp reads both halves of its rows' S
//              to form the row maximum, so the pair never synchronises inside the tile loop;
//   warps 8-11 producer: warp 8+i writes the Q rows of TMEM lanes 32i .. 32i+31 straight from
//              global memory (gathered by perm) into TMEM, and fills the STAGES-deep K/V ring:
//              sparse tiles with 16-byte cp.async copies of the rows named by idx (each lane
//              loads one row index per tile, one tile ahead, and shares it by shuffles), dense
//              tiles with TMA (warp 8 alone, two 64-column boxes per tile).  Both write the
//              128-byte-swizzled K-major layout the MMAs read.  (TMA gather4 was measured
//              three times slower than the cp.async gather for these 128-byte rows.)
//   warp 12    TMEM allocator and the single MMA-issuing thread.
// TMEM (512 columns): S = Q K^T in two 128-column buffers, O (d columns), P (64 columns of bf16
// pairs) and Q (d/2 columns of bf16 pairs).  Both MMAs take A from TMEM (S = Q K^T with A = Q,
// O += P V with A = P), so shared memory only feeds the B operands (K and V); softmax reads S and
// writes P back to TMEM.  The running max is raised lazily (only when it grows by more than
// 2^8), so O is rescaled in TMEM rarely.
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

constexpr int kAttnThreads = 416;
constexpr int kTile = 128;

template <int HD>
struct AttnSmem {
  static constexpr uint32_t TILE_BYTES = kTile * HD * 2;  // K or V tile
  static constexpr int STAGES = HD == 128 ? 3 : 6;
  static constexpr uint32_t K_OFF = 0;
  static constexpr uint32_t V_OFF = K_OFF + STAGES * TILE_BYTES;
  static constexpr uint32_t XCH_OFF = V_OFF + STAGES * TILE_BYTES;  // 2 x 2 x 128 row sums
  static constexpr uint32_t XMX_OFF = XCH_OFF + 4 * kTile * 4;       // 2 x 2 x 128 row maxima
  static constexpr uint32_t FLAG_OFF = XMX_OFF + 4 * kTile * 4;      // 8 softmax-warp counters
  static constexpr uint32_t BAR_OFF = FLAG_OFF + 8 * 4;
  // barriers: q_full, q_empty, k_full[S], v_full[S], kv_empty[S], s_full[2], s_empty[2],
  //           p_full, pv_done, o_empty, drain, pair[4]
  static constexpr int NBAR = 2 + 3 * STAGES + 4 + 1 + 1 + 2 + 4;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
  // The dynamic shared memory window starts 1024-byte aligned (checked at run time), which the
  // 128-byte-swizzle atoms of the tiles at offset 0 rely on.
  static constexpr uint32_t BYTES = MISC_OFF + 16;
  static_assert(BYTES <= 232448, "shared memory budget");
};

// TMEM column map (512 columns allocated)
constexpr uint32_t kTmS = 0;      // two S buffers, 128 columns each
constexpr uint32_t kTmO = 256;    // O, d columns
constexpr uint32_t kTmP = 384;    // P, 64 columns (bf16 pairs)
constexpr uint32_t kTmQ = 448;    // Q, d/2 columns (bf16 pairs)

template <int HD, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem<HD>;
  constexpr int STAGES = L::STAGES;
  constexpr int CHUNKS = HD / 8;                       // 16-byte chunks per row
  constexpr int RPI = 32 / CHUNKS;                     // rows per cp.async instruction
  constexpr uint32_t HALF = kTile * 128;               // bytes per 64-column half of a tile
  constexpr uint32_t IDESC_QK = idesc_bf16(128, 128, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, HD, false, true);
  constexpr bool SPARSE = MODE != kDense;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {  // uniform across the CTA: nothing has started yet
    if (threadIdx.x == 0) raise_status(kStatusBadShape);
    return;
  }
  uint8_t* gptr = smem_raw;

  uint64_t* bars = reinterpret_cast<uint64_t*>(gptr + L::BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* v_full = k_full + STAGES;
  uint64_t* kv_empty = v_full + STAGES;
  uint64_t* s_full = kv_empty + STAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* o_empty = pv_done + 1;
  uint64_t* drain = o_empty + 1;
  uint64_t* pair = drain + 1;       // [4], one per softmax row group (its two warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gptr + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gptr + L::MISC_OFF + 4);
  float* sXch = reinterpret_cast<float*>(gptr + L::XCH_OFF);
  float* sXmx = reinterpret_cast<float*>(gptr + L::XMX_OFF);
  uint32_t* sFlag = reinterpret_cast<uint32_t*>(gptr + L::FLAG_OFF);

  const uint32_t sK = base + L::K_OFF;
  const uint32_t sV = base + L::V_OFF;
  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    mbar_init(q_empty, 1);
    for (int s = 0; s < STAGES; ++s) {
      // sparse: one cp.async arrival per producer thread; dense: one arrival with the expected
      // bytes, which the TMA then completes
      mbar_init(k_full + s, SPARSE ? 128 : 1);
      mbar_init(v_full + s, SPARSE ? 128 : 1);
      mbar_init(kv_empty + s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, 256);
    }
    mbar_init(p_full, 256);
    mbar_init(pv_done, 1);
    mbar_init(o_empty, 256);
    mbar_init(drain, 1);
    for (int g = 0; g < 4; ++g) mbar_init(pair + g, 64);
    for (int w = 0; w < 8; ++w) sFlag[w] = 0;
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int T = p.kv_tiles;

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------------ producer
    const int pw = warp - 8;                 // == warp % 4: owns TMEM lanes 32*pw .. +31
    const int my_row = pw * 32 + lane;       // tile row of this lane
    const uint32_t tQ = tmem + (static_cast<uint32_t>(pw * 32) << 16) + kTmQ;
    const int sub = lane / CHUNKS, c = lane % CHUNKS;  // cp.async lane mapping (sparse)
    uint32_t kv_it = 0, u_it = 0;
    for (int unit = blockIdx.x; unit < p.num_units; unit += gridDim.x, ++u_it) {
      const int bh = unit / p.units_per_head;
      const int ut = unit - bh * p.units_per_head;
      const size_t head_off = static_cast<size_t>(bh) * p.N;
      const int32_t* idx_row = SPARSE ? p.idx + (static_cast<size_t>(bh) * p.G + ut) * p.k : nullptr;
      // this lane's Q row (and first KV index), loaded before waiting for the previous unit's
      // last QK^T
      int q;
      bool qok;
      if (SPARSE) {
        qok = my_row < p.C;
        q = qok ? p.perm[head_off + static_cast<size_t>(ut) * p.C + my_row] : 0;
        if (qok && static_cast<unsigned>(q) >= static_cast<unsigned>(p.N)) {
          raise_status(kStatusBadIndex);
          qok = false;
        }
      } else {
        q = ut * kTile + my_row;
        qok = q < p.N;
      }
      int nidx = -1;
      if (SPARSE && my_row < p.kv_count) nidx = idx_row[my_row];
      uint32_t qreg[HD / 2];
      {
        const uint4* src = reinterpret_cast<const uint4*>(p.Q + (head_off + (qok ? q : 0)) * HD);
#pragma unroll
        for (int i = 0; i < HD / 8; ++i) {
          const uint4 v = qok ? src[i] : make_uint4(0u, 0u, 0u, 0u);
          qreg[4 * i] = v.x;
          qreg[4 * i + 1] = v.y;
          qreg[4 * i + 2] = v.z;
          qreg[4 * i + 3] = v.w;
        }
      }
      if (!mbar_wait_warp(q_empty, (u_it & 1) ^ 1, abort_flag)) break;
      tc_fence_after();
      if (HD == 128) {
        tmem_st64(tQ, qreg);
      } else {
        tmem_st32(tQ, qreg);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(q_full);
      bool okp = true;
      if (SPARSE) {
        // ---- gathered tiles: every producer lane copies 16-byte chunks with cp.async.  Lane
        // `lane` of warp pw copies chunk c of rows pw*32 + it*RPI + sub (it = 0 .. 32/RPI-1):
        // its shared-memory offsets are the same for every tile, and a row's global offset is
        // computed once and reused for K and V.
        constexpr int NIT = 32 / RPI;
        uint32_t soff[NIT];
#pragma unroll
        for (int it = 0; it < NIT; ++it) soff[it] = sw128_offset(pw * 32 + it * RPI + sub, c, kTile);
        for (int j = 0; j < T; ++j, ++kv_it) {
          const uint32_t st = kv_it % STAGES;
          int cur = nidx;
          if (cur != -1 && static_cast<unsigned>(cur) >= static_cast<unsigned>(p.N)) {
            raise_status(kStatusBadIndex);
            cur = -1;
          }
          const int pos = (j + 1) * kTile + my_row;
          nidx = (j + 1 < T && pos < p.kv_count) ? idx_row[pos] : -1;  // prefetch the next tile
          // element offsets of this lane's rows (the zero-filled chunks read nothing)
          size_t goff[NIT];
          uint32_t gbytes[NIT];
#pragma unroll
          for (int it = 0; it < NIT; ++it) {
            const int kv = __shfl_sync(0xffffffffu, cur, it * RPI + sub);
            gbytes[it] = kv >= 0 ? 16u : 0u;
            goff[it] = (head_off + static_cast<size_t>(kv >= 0 ? kv : 0)) * HD + c * 8;
          }
          if (!mbar_wait_warp(kv_empty + st, ((kv_it / STAGES) & 1) ^ 1, abort_flag)) {
            okp = false;
            break;
          }
          const uint32_t dK = sK + st * L::TILE_BYTES, dV = sV + st * L::TILE_BYTES;
          // K rows, then V rows, each followed by its own arrival so QK^T can start early.
#pragma unroll
          for (int it = 0; it < NIT; ++it) cp_async16(dK + soff[it], p.K + goff[it], gbytes[it]);
          cp_async_arrive(k_full + st);
#pragma unroll
          for (int it = 0; it < NIT; ++it) cp_async16(dV + soff[it], p.V + goff[it], gbytes[it]);
          cp_async_arrive(v_full + st);
        }
      } else if (pw == 0) {
        // ---- dense tiles: warp 8 alone streams two 64-column boxes per tile with TMA (rows
        // past the tensor are zero-filled; rows of the next head in a last partial tile are
        // masked by the softmax)
        for (int j = 0; j < T; ++j, ++kv_it) {
          const uint32_t st = kv_it % STAGES;
          if (!mbar_wait_warp(kv_empty + st, ((kv_it / STAGES) & 1) ^ 1, abort_flag)) {
            okp = false;
            break;
          }
          if (lane == 0) {
#pragma unroll
            for (int which = 0; which < 2; ++which) {
              const CUtensorMap* map = which == 0 ? &tmK : &tmV;
              uint64_t* full = (which == 0 ? k_full : v_full) + st;
              const uint32_t dst = (which == 0 ? sK : sV) + st * L::TILE_BYTES;
              mbar_arrive_expect_tx(full, L::TILE_BYTES);
#pragma unroll
              for (int h = 0; h < HD / 64; ++h)
                tma_load_2d(dst + h * HALF, map, h * 64, static_cast<int>(head_off) + j * kTile, full);
            }
          }
          __syncwarp();
        }
      }
      if (!okp) break;
    }
    cp_async_wait_all();
  } else if (warp == 12) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t tS = tmem + kTmS, tO = tmem + kTmO, tP = tmem + kTmP, tQ = tmem + kTmQ;
      // Descriptors of stage 0; a stage and a k-step only move the start-address field (bits
      // 0-13, in 16-byte units), which never carries: shared addresses stay below 256 KiB.
      const uint64_t dK0 = desc_sw128(sK, 16, 1024);
      const uint64_t dV0 = desc_sw128(sV, HALF, 1024);
      constexpr uint64_t kStageStep = L::TILE_BYTES >> 4;
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
          const uint64_t dK = dK0 + st * kStageStep;
          const uint32_t dS = tS + b * 128;
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks)
            mma_bf16_ts(dS, tQ + ks * 8, dK + (((ks >> 2) * HALF + (ks & 3) * 32) >> 4), IDESC_QK, ks > 0 ? 1u : 0u);
          mma_commit(s_full + b);
          return true;
        };
        auto issue_pv = [&](int j) -> bool {
          const uint32_t it = kv_base + j, st = it % STAGES;
          const uint32_t si = s_base + j;
          if (!mbar_wait(p_full, si & 1, abort_flag)) return false;
          if (!mbar_wait(v_full + st, (it / STAGES) & 1, abort_flag)) return false;
          if (j == 0 && !mbar_wait(o_empty, (u_it & 1) ^ 1, abort_flag)) return false;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t dV = dV0 + st * kStageStep;
          mma_bf16_ts(tO, tP, dV, IDESC_PV, j > 0 ? 1u : 0u);
#pragma unroll
          for (int ks = 1; ks < kTile / 16; ++ks) mma_bf16_ts(tO, tP + ks * 8, dV + ks * (2048 >> 4), IDESC_PV, 1u);
          mma_commit(kv_empty + st);
          mma_commit(pv_done);
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
    const int rg = warp & 3, ch = warp >> 2;  // row group, column half
    const int row = rg * 32 + lane;           // tile row == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(rg * 32) << 16;
    const uint32_t tS = tmem + lane_base + kTmS + ch * 64;
    const uint32_t tO = tmem + lane_base + kTmO + ch * (HD / 2);
    const uint32_t tP = tmem + lane_base + kTmP + ch * 32;
    const float sl2 = p.scale_log2;
    uint32_t s_base = 0, u_it = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x) {
      const int bh = unit / p.units_per_head;
      const int ut = unit - bh * p.units_per_head;
      float m_used = -INFINITY, l_part = 0.f;
      for (int j = 0; j < T; ++j) {
        const uint32_t si = s_base + j, b = si & 1;
        if (!mbar_wait_warp(s_full + b, (si >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        const int nvalid = min(kTile, p.kv_count - j * kTile);  // valid columns of the tile
        const int valid = nvalid - ch * 64;                      // ... of my half
        tmem_ld32(tS + b * 128 + 0, sr);
        tmem_ld32(tS + b * 128 + 32, sr + 32);
        tmem_ld_wait_regs(sr);
        reg_fence32(sr + 32);
        tc_fence_before();
        mbar_arrive(s_empty + b);
        float mx = -INFINITY;
        if (nvalid == kTile) {
#pragma unroll
          for (int c = 0; c < 64; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) mx = fmaxf(mx, c < valid ? __uint_as_float(sr[c]) : -INFINITY);
        }
        // row maximum across the two column halves: publish mine, read the partner's (slot
        // parity alternates per tile; each warp's counter says which tile it has published)
        {
          float* xm = sXmx + (si & 1) * 2 * kTile;
          xm[ch * kTile + row] = mx;
          __syncwarp();
          if (lane == 0) st_release_u32(sFlag + warp, si + 1);
          if (!flag_wait_warp(sFlag + (warp ^ 4), si + 1, abort_flag)) { ok = false; break; }
          mx = fmaxf(mx, xm[(ch ^ 1) * kTile + row]);
        }
        const float m_tile = mx * sl2;
        float m_new = m_used, alpha = 1.f;
        const bool raise = m_tile > m_used + 8.f;
        if (raise) {
          m_new = m_tile;
          alpha = fast_exp2(m_used - m_new);  // 0 on the first tile
        }
        float rs0 = 0.f, rs1 = 0.f;
        uint32_t pw[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c = 2 * i;
          float e0 = fast_exp2(fmaf(__uint_as_float(sr[c]), sl2, -m_new));
          float e1 = fast_exp2(fmaf(__uint_as_float(sr[c + 1]), sl2, -m_new));
          if (nvalid != kTile) {
            e0 = c < valid ? e0 : 0.f;
            e1 = c + 1 < valid ? e1 : 0.f;
          }
          rs0 += e0;
          rs1 += e1;
          pw[i] = pack_bf16x2(e0, e1);
        }
        l_part = l_part * alpha + (rs0 + rs1);
        m_used = m_new;
        // P (and O) are free once PV of the previous tile has completed
        if (j > 0) {
          if (!mbar_wait_warp(pv_done, (si - 1) & 1, abort_flag)) { ok = false; break; }
          tc_fence_after();
          // tcgen05.ld/st are warp-collective: rescale the warp's rows if any of them needs it
          // (alpha is 1 for rows whose max did not move)
          if (__any_sync(0xffffffffu, raise)) {
#pragma unroll 1
            for (int c0 = 0; c0 < HD / 2; c0 += 32) {
              uint32_t o[32];
              tmem_ld32(tO + c0, o);
              tmem_ld_wait_regs(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(tO + c0, o);
            }
          }
        }
        tmem_st32(tP, pw);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok) break;
      const uint32_t si_last = s_base + T - 1;
      if (!mbar_wait_warp(pv_done, si_last & 1, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // row sum across the two column halves: exchange through shared memory around a bounded
      // mbarrier rendezvous of the row group's two warps (slot parity alternates per unit)
      float* xch = sXch + (u_it & 1) * 2 * kTile;
      xch[ch * kTile + row] = l_part;
      mbar_arrive(pair + rg);
      if (!mbar_wait_warp(pair + rg, u_it & 1, abort_flag)) { ok = false; break; }
      const float l_sum = l_part + xch[(ch ^ 1) * kTile + row];
      // ---- epilogue: this thread's output row, columns [ch*HD/2, (ch+1)*HD/2)
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
      const size_t rbase = (static_cast<size_t>(bh) * p.N + q) * HD + ch * (HD / 2);
#pragma unroll 1
      for (int c0 = 0; c0 < HD / 2; c0 += 32) {
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
      if (MODE == kDense && ch == 0 && live && p.lse != nullptr) {
        p.lse[static_cast<size_t>(bh) * p.N + q] = (m_used + __log2f(l_sum)) * 0.69314718055994531f;
      }
      tc_fence_before();
      mbar_arrive(o_empty);
      s_base += T;
      ++u_it;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mcs
