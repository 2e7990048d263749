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
// One CTA per SM, persistent over work units (one 128-row query tile each).  The keys of a unit
// come in 128-key stages that alternate between two independent online-softmax streams A (even
// stages) and B (odd stages): split-K inside the CTA.  Each stream has its own S (whose first
// half the stream's P overwrites in place), running max and sum, and O accumulator in TMEM; the
// two are merged once per unit in the epilogue,
//     O = (O_A 2^(m_A-m) + O_B 2^(m_B-m)) / (l_A 2^(m_A-m) + l_B 2^(m_B-m)),  m = max(m_A, m_B).
// While one stream's softmax runs, the tensor core works on the other stream's products, so
// the hand-offs between the roles (S ready, P ready, PV done) do not idle it.
// Warp roles (512 threads, four warpgroups; setmaxnreg gives the softmax warpgroups 192
// registers a thread, the producers 80 and the MMA warpgroup 48):
//   warps 0-7   softmax + epilogue: warp w owns tile rows 32*(w%4) .. +31 (its TMEM lanes) of
//               stream w/4, one whole S row per thread, loaded from TMEM in one round trip (four
//               32-column loads in flight, one wait: a round trip costs about 400 cycles, so
//               one per stage instead of four); in the epilogue it writes output columns
//               (w/4)*d/2 .. +d/2 of its rows from both streams' O, read in one round trip,
//               with the row's R (or O_full) loads issued as its last stage ends;
//   warps 8-11  producer: the unit's Q rows (gathered by perm) and the K and V rings, with
//               16-byte cp.async copies (Q; the K/V rows named by idx in the sparse modes: each
//               lane loads one row index per stage, one stage ahead, and shares it by shuffles)
//               or TMA (dense K/V, warp 8 alone, two 64-column boxes per tile), all in the
//               128-byte-swizzled K-major layout the MMAs read.  (TMA gather4 was measured three
//               times slower than the cp.async gather for these 128-byte rows.)
//   warp 12     TMEM allocator and MMA issuer: S_x = Q K^T with both operands in shared memory,
//               O_x += P_x V with P_x from TMEM.  The whole warp runs the issuing loop and lane 0
//               issues, so descriptors and counters are warp-uniform values (a single-thread
//               loop measured 16-27 % slower on this chain).  The MMAs execute in issue order,
//               so a stream's next S may be issued right behind the PV that reads its P from
//               the same columns.  The softmax hands P over in two parts: the PV of a stage's
//               first 96 keys runs while the softmax finishes the last 32.  Warps 13-15 only
//               complete the warpgroup.
// TMEM (512 columns): O_A, O_B (d columns each) and S_A, S_B (128 columns each).
// Softmax per stream and row: the first stage of a unit takes the exact row maximum as its
// reference m; later stages take one pass, P = 2^(s scale log2e - m), which may exceed 1.  A
// stage whose P sums past 2^16 raises m at the stream's next stage (after the previous PV, so O
// and l are rescaled in TMEM rarely); a chunk whose P would sum past 2^64 or overflow raises m
// at once by whole octaves and rescales the stage's stored P exactly (once the first part of P
// has been handed over, that part is rescaled inside O after its PV has completed).
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
  unsigned long long wait_ns;    // bound on any single wait of this launch (nanoseconds)
  const uint32_t* hold;          // test hook (normally NULL): wait for *hold != 0 before any MMA
  int units_per_head;            // dense: ceil(N/128); sparse: G
  int kv_tiles;                  // dense: ceil(N/128); sparse: ceil(k/128)
  int kv_count;                  // dense: N; sparse: k
  int num_units;                 // BH * units_per_head
  float scale_log2;              // scale * log2(e)
  int store_out;                 // kDense: 0 = LSE only
};

// Four warpgroups: softmax of stream A (warps 0-3) and of stream B (4-7), producers (8-11), the
// MMA issuer (warp 12; warps 13-15 only complete the warpgroup).  The 65536 registers of the
// launch (512 threads x 128) are split 192 / 192 / 80 / 48 per thread by setmaxnreg, so that a
// softmax thread holds a whole 128-column S row and its 64 packed P words in registers.
constexpr int kAttnThreads = 512;
constexpr uint32_t kRegsSoftmax = 192, kRegsProducer = 80, kRegsMma = 48;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsProducer + 128 * kRegsMma <= 512 * 128,
              "warpgroup register split exceeds the launch's registers");
constexpr int kTile = 128;
// P is handed to the tensor core in two parts: its first kPSplit 32-key chunks, then the rest
// (three of four measured faster than two: the PV of 96 keys runs under the last chunk's
// exponentials)
constexpr int kPSplit = 3;
static_assert(kPSplit >= 1 && kPSplit < kTile / 32, "P hand-over split");

template <int HD>
struct AttnSmem {
  static constexpr uint32_t TILE_BYTES = kTile * HD * 2;  // Q, K or V tile
  static constexpr int KST = HD == 128 ? 3 : 6;           // K ring
  static constexpr int VST = HD == 128 ? 3 : 6;           // V ring
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = Q_OFF + TILE_BYTES;
  static constexpr uint32_t V_OFF = K_OFF + KST * TILE_BYTES;
  static constexpr uint32_t XCH_OFF = V_OFF + VST * TILE_BYTES;  // 2 streams x 128 rows x (m, l)
  static constexpr uint32_t BAR_OFF = XCH_OFF + 2 * kTile * 8;
  // barriers: q_full, q_empty, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], then per
  //           stream s_full[2], p_full[2], pv_done[2]; o_empty, drain, pair[4]; per stream
  //           p_half[2], pvlo_done[2]
  static constexpr int NBAR = 2 + 2 * KST + 2 * VST + 6 + 2 + 4 + 4;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
  // The dynamic shared memory window starts 1024-byte aligned (checked at run time), which the
  // 128-byte-swizzle atoms of the tiles at offset 0 rely on.
  static constexpr uint32_t BYTES = MISC_OFF + 16;
  static_assert(BYTES <= 232448, "shared memory budget");
};

// TMEM column map (512 columns allocated)
constexpr uint32_t kTmO = 0;      // O_A at 0, O_B at d: d columns each
constexpr uint32_t kTmS = 256;    // S_A at 256, S_B at 384: 128 columns each; P_x in the first 64

template <int HD, int MODE>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem<HD>;
  constexpr int KST = L::KST, VST = L::VST;
  constexpr int CHUNKS = HD / 8;                       // 16-byte chunks per row
  constexpr int RPI = 32 / CHUNKS;                     // rows per cp.async instruction
  constexpr int NIT = 32 / RPI;                        // cp.async instructions per warp and tile
  constexpr uint32_t HALF = kTile * 128;               // bytes per 64-column half of a tile
  constexpr uint32_t IDESC_QK = idesc_bf16(128, kTile, false, false);
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
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;  // [2], per stream
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_empty = pv_done + 2;
  uint64_t* drain = o_empty + 1;
  uint64_t* pair = drain + 1;        // [4], one per row group (its two warps)
  uint64_t* p_half = pair + 4;       // [2], per stream: P of the stage's first part stored
  uint64_t* pvlo_done = p_half + 2;  // [2], per stream: the PV of that part has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gptr + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gptr + L::MISC_OFF + 4);
  float2* sXch = reinterpret_cast<float2*>(gptr + L::XCH_OFF);

  const uint32_t sQ = base + L::Q_OFF;
  const uint32_t sK = base + L::K_OFF;
  const uint32_t sV = base + L::V_OFF;
  const int warp = warp_id();
  const int lane = lane_id();
  const uint64_t wl = p.wait_ns;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    mbar_init(q_empty, 1);
    // sparse: one cp.async arrival per producer thread; dense: one arrival with the expected
    // bytes, which the TMA then completes
    for (int s = 0; s < KST; ++s) {
      mbar_init(k_full + s, SPARSE ? 128 : 1);
      mbar_init(k_empty + s, 128);  // the consuming stream's softmax threads, once S is ready
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(v_full + s, SPARSE ? 128 : 1);
      mbar_init(v_empty + s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(s_full + x, 1);
      mbar_init(p_full + x, 128);
      mbar_init(pv_done + x, 1);
      mbar_init(p_half + x, 128);
      mbar_init(pvlo_done + x, 1);
    }
    mbar_init(o_empty, 256);
    mbar_init(drain, 1);
    for (int g = 0; g < 4; ++g) mbar_init(pair + g, 64);
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

  const int T = p.kv_tiles;  // stages per unit; stage j belongs to stream j & 1

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------------ producer
    regs_to<kRegsProducer, 65536 / kAttnThreads>();
    const int pw = warp - 8;
    const int my_row = pw * 32 + lane;                 // tile row of this lane
    const int sub = lane / CHUNKS, c = lane % CHUNKS;  // cp.async lane mapping
    // Lane `lane` of warp pw copies chunk c of rows pw*32 + it*RPI + sub (it = 0 .. NIT-1): its
    // shared-memory offsets are the same for every tile.
    uint32_t soff[NIT];
#pragma unroll
    for (int it = 0; it < NIT; ++it) soff[it] = sw128_offset(pw * 32 + it * RPI + sub, c, kTile);
    uint32_t kv_it = 0, u_it = 0;
    uint32_t k_issued = 0, v_issued = 0;  // TMA loads issued into the K and V rings (dense)
    bool okp = true;
    for (int unit = blockIdx.x; unit < p.num_units && okp; unit += gridDim.x, ++u_it) {
      const int bh = unit / p.units_per_head;
      const int ut = unit - bh * p.units_per_head;
      const size_t head_off = static_cast<size_t>(bh) * p.N;
      const int32_t* idx_row = SPARSE ? p.idx + (static_cast<size_t>(bh) * p.G + ut) * p.k : nullptr;
      // this lane's Q row and first KV index
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
      const int qrow = qok ? q : -1;
      int nidx = -1;
      if (SPARSE && my_row < p.kv_count) nidx = idx_row[my_row];
      // ---- Q tile (after the previous unit's last QK^T has read it)
      if (!mbar_wait_warp(q_empty, (u_it & 1) ^ 1, abort_flag, wl)) { okp = false; break; }
#pragma unroll
      for (int it = 0; it < NIT; ++it) {
        const int r = __shfl_sync(0xffffffffu, qrow, it * RPI + sub);
        cp_async16(sQ + soff[it], p.Q + (head_off + static_cast<size_t>(r >= 0 ? r : 0)) * HD + c * 8,
                   r >= 0 ? 16u : 0u);
      }
      cp_async_arrive(q_full);
      if (SPARSE && qok) {
        // the row of R (reuse) or O_full (residual) that the epilogue of this unit combines
        const __nv_bfloat16* ep = MODE == kReuse ? p.R_in : p.O_full;
        if (ep != nullptr) {
#pragma unroll
          for (int b = 0; b < HD * 2; b += 128) prefetch_l2(reinterpret_cast<const uint8_t*>(ep + (head_off + q) * HD) + b);
        }
      }
      if (SPARSE) {
        // ---- gathered K/V tiles; a row's global offset is computed once for K and V
        const __nv_bfloat16* Kh = p.K + head_off * HD;
        const __nv_bfloat16* Vh = p.V + head_off * HD;
        for (int j = 0; j < T; ++j, ++kv_it) {
          const uint32_t ks = kv_it % KST, vs = kv_it % VST;
          int cur = nidx;
          if (cur != -1 && static_cast<unsigned>(cur) >= static_cast<unsigned>(p.N)) {
            raise_status(kStatusBadIndex);
            cur = -1;
          }
          const int pos = (j + 1) * kTile + my_row;
          nidx = (j + 1 < T && pos < p.kv_count) ? idx_row[pos] : -1;  // prefetch the next stage
          // element offsets within the head (< N*d, checked on the host to fit 32 bits)
          uint32_t goff[NIT];
          uint32_t gbytes[NIT];
#pragma unroll
          for (int it = 0; it < NIT; ++it) {
            const int kv = __shfl_sync(0xffffffffu, cur, it * RPI + sub);
            gbytes[it] = kv >= 0 ? 16u : 0u;
            goff[it] = static_cast<uint32_t>(kv >= 0 ? kv : 0) * HD + c * 8;
          }
          if (!mbar_wait_warp(k_empty + ks, ((kv_it / KST) & 1) ^ 1, abort_flag, wl)) { okp = false; break; }
          const uint32_t dK = sK + ks * L::TILE_BYTES;
#pragma unroll
          for (int it = 0; it < NIT; ++it) cp_async16(dK + soff[it], Kh + goff[it], gbytes[it]);
          cp_async_arrive(k_full + ks);
          if (!mbar_wait_warp(v_empty + vs, ((kv_it / VST) & 1) ^ 1, abort_flag, wl)) { okp = false; break; }
          const uint32_t dV = sV + vs * L::TILE_BYTES;
#pragma unroll
          for (int it = 0; it < NIT; ++it) cp_async16(dV + soff[it], Vh + goff[it], gbytes[it]);
          cp_async_arrive(v_full + vs);
        }
      } else if (pw == 0) {
        // ---- dense tiles: warp 8 alone streams two 64-column boxes per tile with TMA (rows
        // past the tensor are zero-filled; rows of the next head in a last partial tile are
        // masked by the softmax)
        for (int j = 0; j < T; ++j, ++kv_it) {
          const uint32_t ks = kv_it % KST, vs = kv_it % VST;
          const int row0 = static_cast<int>(head_off) + j * kTile;
          if (!mbar_wait_warp(k_empty + ks, ((kv_it / KST) & 1) ^ 1, abort_flag, wl)) { okp = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(k_full + ks, L::TILE_BYTES);
#pragma unroll
            for (int h = 0; h < HD / 64; ++h) tma_load_2d(sK + ks * L::TILE_BYTES + h * HALF, &tmK, h * 64, row0, k_full + ks);
          }
          ++k_issued;
          __syncwarp();
          if (!mbar_wait_warp(v_empty + vs, ((kv_it / VST) & 1) ^ 1, abort_flag, wl)) { okp = false; break; }
          if (lane == 0) {
            mbar_arrive_expect_tx(v_full + vs, L::TILE_BYTES);
#pragma unroll
            for (int h = 0; h < HD / 64; ++h) tma_load_2d(sV + vs * L::TILE_BYTES + h * HALF, &tmV, h * 64, row0, v_full + vs);
          }
          ++v_issued;
          __syncwarp();
        }
      } else {
        kv_it += T;
      }
    }
    cp_async_wait_all();
    if (!SPARSE && pw == 0 && !okp) {
      // after an abort, the TMA loads already issued land before the CTA releases its shared
      // memory: the last load into each slot completes the phase counted for it (on a normal
      // exit every load has been consumed, so there is nothing to wait for)
      for (uint32_t s = 0; s < static_cast<uint32_t>(KST) && s < k_issued; ++s) {
        const uint32_t last = k_issued - 1 - ((k_issued - 1 + KST - s) % KST);
        mbar_drain(k_full + s, (last / KST) & 1);
      }
      for (uint32_t s = 0; s < static_cast<uint32_t>(VST) && s < v_issued; ++s) {
        const uint32_t last = v_issued - 1 - ((v_issued - 1 + VST - s) % VST);
        mbar_drain(v_full + s, (last / VST) & 1);
      }
    }
  } else if (warp >= 12) {
    // ------------------------------------------------------------------ MMA issuer
    regs_to<kRegsMma, 65536 / kAttnThreads>();
    if (warp == 12) {
      // The whole warp runs this loop (its waits agree warp-wide) and lane 0 issues each
      // tcgen05 instruction, so the descriptors and counters are warp-uniform values.
      // Descriptors of slot 0; a slot and a k-step only move the start-address field (bits
      // 0-13, in 16-byte units), which never carries: shared addresses stay below 256 KiB.
      const uint64_t dQ = desc_sw128(sQ, 16, 1024);
      const uint64_t dK0 = desc_sw128(sK, 16, 1024);
      const uint64_t dV0 = desc_sw128(sV, HALF, 1024);
      constexpr uint64_t kSlotStep = L::TILE_BYTES >> 4;
      uint32_t kv_base = 0, u_it = 0;
      uint32_t sc0 = 0, sc1 = 0;  // PVs issued per stream (barrier phases)
      bool ok = true;
      if (p.hold != nullptr) {
        // a flag in global memory that the caller may never set: the wait for it runs out like
        // any other, which makes every role of the CTA take its abort path
        if (lane == 0) {
          const uint64_t t0 = globaltimer_ns();
          while (ld_acquire_gpu_u32(p.hold) == 0u) {
            if (globaltimer_ns() - t0 > wl) {
              raise_status(kStatusTimeout);
              *abort_flag = 1;
              ok = false;
              break;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      }
      for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x, ++u_it) {
        ok = mbar_wait_warp(q_full, u_it & 1, abort_flag, wl);
        if (!ok) break;
        fence_proxy_async_smem();  // Q arrives by cp.async (generic proxy) -> tensor-core reads
        // The tensor core keeps almost no queue: any wait, fence or branch between two MMAs idles
        // it.  So every step first waits for all it needs, then issues its MMAs back to back: PV
        // of stage j and the QK^T of stage j+2 (same stream, so the QK^T overwrites S_x right
        // behind the PV that reads P_x from it: the MMAs of one CTA execute in issue order).
        auto qk_mmas = [&](int j) {
          const uint32_t it = kv_base + j, ks = it % KST;
          const uint64_t dK = dK0 + ks * kSlotStep;
          const uint32_t dS = tmem + kTmS + (j & 1) * kTile;
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint64_t koff = ((kk >> 2) * HALF + (kk & 3) * 32) >> 4;
            mma_bf16_ss_warp(dS, dQ + koff, dK + koff, IDESC_QK, kk > 0 ? 1u : 0u);
          }
        };
        auto wait_k = [&](int j) -> bool {
          const uint32_t it = kv_base + j;
          return mbar_wait_warp(k_full + it % KST, (it / KST) & 1, abort_flag, wl);
        };
        // prologue: S of the first stage of each stream
        ok = wait_k(0) && (T < 2 || wait_k(1));
        if (!ok) break;
        if (SPARSE) fence_proxy_async_smem();  // gathered K arrives by cp.async
        qk_mmas(0);
        mma_commit_warp(s_full + 0);
        if (T > 1) {
          qk_mmas(1);
          mma_commit_warp(s_full + 1);
        }
        if (T <= 2) mma_commit_warp(q_empty);
        for (int j = 0; j < T && ok; ++j) {
          const int x = j & 1;
          const uint32_t it = kv_base + j, vs = it % VST;
          const bool next = j + 2 < T;
          // the PV of the stage's first 32 * kPSplit keys as soon as their P is stored, the rest
          // (and the stream's next QK^T) once the whole P is
          ok = mbar_wait_warp(p_half + x, (x ? sc1 : sc0) & 1, abort_flag, wl) &&
               mbar_wait_warp(v_full + vs, (it / VST) & 1, abort_flag, wl) &&
               (j != 0 || mbar_wait_warp(o_empty, (u_it & 1) ^ 1, abort_flag, wl));
          if (!ok) break;
          if (SPARSE) fence_proxy_async_smem();  // gathered V arrives by cp.async
          tc_fence_after();                      // P_x was written by tcgen05.st of the softmax
          const uint64_t dV = dV0 + vs * kSlotStep;
          const uint32_t tO = tmem + kTmO + x * HD, tP = tmem + kTmS + x * kTile;
          const bool first = j < 2;  // the stream's first stage of the unit overwrites O_x
#pragma unroll
          for (int kk = 0; kk < 2 * kPSplit; ++kk)
            mma_bf16_ts_warp(tO, tP + kk * 8, dV + kk * (2048 >> 4), IDESC_PV, (!first || kk > 0) ? 1u : 0u);
          mma_commit_warp(pvlo_done + x);
          ok = mbar_wait_warp(p_full + x, (x ? sc1 : sc0) & 1, abort_flag, wl) && (!next || wait_k(j + 2));
          if (!ok) break;
          if (SPARSE) fence_proxy_async_smem();  // gathered K arrives by cp.async
          tc_fence_after();
#pragma unroll
          for (int kk = 2 * kPSplit; kk < kTile / 16; ++kk)
            mma_bf16_ts_warp(tO, tP + kk * 8, dV + kk * (2048 >> 4), IDESC_PV, 1u);
          mma_commit_warp(pv_done + x);
          mma_commit_warp(v_empty + vs);
          if (x) ++sc1;
          else ++sc0;
          if (next) {
            qk_mmas(j + 2);
            mma_commit_warp(s_full + x);
            if (j + 3 == T) mma_commit_warp(q_empty);
          }
        }
        kv_base += T;
      }
      // drain: every MMA issued above has completed before TMEM is released
      mma_commit_warp(drain);
      mbar_drain(drain, 0);
    }  // warps 13-15 only complete the warpgroup
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    regs_to<kRegsSoftmax, 65536 / kAttnThreads>();
    const int rg = warp & 3, x = warp >> 2;  // row group, stream
    const int row = rg * 32 + lane;          // tile row == TMEM lane
    const uint32_t lane_base = static_cast<uint32_t>(rg * 32) << 16;
    const uint32_t tS = tmem + lane_base + kTmS + x * kTile;  // S_x; P_x in its first 64 columns
    const uint32_t tOx = tmem + lane_base + kTmO + x * HD;
    const float sl2 = p.scale_log2;
    uint32_t sc = 0;        // stages of this stream processed (barrier phases)
    uint32_t kv_base = 0;   // stages of earlier units
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x, kv_base += T) {
      const int bh = unit / p.units_per_head;
      const int ut = unit - bh * p.units_per_head;
      float m_used = -INFINITY, l_part = 0.f;
      float m_pend = -INFINITY;  // a raise of the reference decided by the stream's previous stage
      // the output row of this thread (its query), read now so that the epilogue does not wait
      int qrow;
      bool live;
      if (SPARSE) {
        live = row < p.C;
        qrow = live ? p.perm[static_cast<size_t>(bh) * p.N + static_cast<size_t>(ut) * p.C + row] : 0;
      } else {
        qrow = ut * kTile + row;
        live = qrow < p.N;
      }
      for (int j = x; j < T; j += 2, ++sc) {
        if (!mbar_wait_warp(s_full + x, sc & 1, abort_flag, wl)) { ok = false; break; }
        // the QK^T that wrote S has read its K slot: hand the slot back to the producer
        mbar_arrive(k_empty + (kv_base + j) % KST);
        tc_fence_after();
        const int valid = p.kv_count - j * kTile;  // valid keys of the stage (>= 1)
        // O_x times alpha (1 for rows whose reference does not move); tcgen05.ld/st are
        // warp-collective, so the whole warp runs it when any of its rows needs it
        auto rescale_o = [&](float alpha) {
#pragma unroll 1
          for (int c0 = 0; c0 < HD; c0 += 32) {
            uint32_t o[32];
            tmem_ld32(tOx + c0, o);
            tmem_ld_wait_regs(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tOx + c0, o);
          }
        };
        // the P of the stage's first kPSplit chunks is stored: its PV may start
        auto signal_half = [&]() {
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(p_half + x);
        };
        // P = exp2(S*scale*log2e - m) of one 32-key chunk (S in sr) in bf16 pairs, and its sums
        // over the even and over the odd keys (fp32 pairs: one packed instruction for two keys)
        auto chunk_exps = [&](const uint32_t* sr, int q, float m, uint32_t* pw, float2& cs) {
          cs = make_float2(0.f, 0.f);
          const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m, -m);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = 32 * q + 2 * i;
            const float2 xv =
                __ffma2_rn(make_float2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sc2, nm2);
            float2 e = make_float2(fast_exp2(xv.x), fast_exp2(xv.y));
            if (valid < kTile) {
              e.x = c < valid ? e.x : 0.f;
              e.y = c + 1 < valid ? e.y : 0.f;
            }
            cs = __fadd2_rn(cs, e);
            pw[i] = pack_bf16x2(e.x, e.y);
          }
        };
        // The whole row of S in one TMEM round trip (four loads in flight, one wait); the P of
        // chunk q goes to columns [16q, 16q+16) of S_x (already in registers) as it is made.
        uint32_t sr[128];
        tmem_ld32(tS, sr);
        tmem_ld32(tS + 32, sr + 32);
        tmem_ld32(tS + 64, sr + 64);
        tmem_ld32(tS + 96, sr + 96);
        tmem_ld_wait_regs(sr);
        reg_fence32(sr + 32);
        reg_fence32(sr + 64);
        reg_fence32(sr + 96);
        float2 rs = make_float2(0.f, 0.f);
        if (j < 2) {
          // the stream's first stage of the unit: the exact row maximum first, then P
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
          if (valid >= kTile) {
#pragma unroll
            for (int c = 0; c < kTile; ++c) m4[c & 3] = fmaxf(m4[c & 3], __uint_as_float(sr[c]));
          } else {
#pragma unroll
            for (int c = 0; c < kTile; ++c) m4[c & 3] = fmaxf(m4[c & 3], c < valid ? __uint_as_float(sr[c]) : -INFINITY);
          }
          m_used = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;  // O_x is fresh
#pragma unroll
          for (int q = 0; q < kTile / 32; ++q) {
            uint32_t pw[16];
            float2 cs;
            chunk_exps(sr + 32 * q, q, m_used, pw, cs);
            rs = __fadd2_rn(rs, cs);
            tmem_st16(tS + 16 * q, pw);
            if (q == kPSplit - 1) signal_half();
          }
          m_pend = -INFINITY;
        } else {
          // later stages, one pass: P against the running reference m_used, which need not be
          // the row maximum (P may exceed 1; bf16 keeps its relative precision and fp32 O and l
          // have the range).  A stage whose P summed to more than 2^16 raised the reference for
          // this stage, applied here once the stream's previous PV has completed so that O_x and
          // l follow; a chunk whose P would sum past 2^64 (or overflow) raises it at once.
          if (__any_sync(0xffffffffu, m_pend > m_used)) {
            if (!mbar_wait_warp(pv_done + x, (sc - 1) & 1, abort_flag, wl)) { ok = false; break; }
            tc_fence_after();
            const float alpha = m_pend > m_used ? fast_exp2(m_used - m_pend) : 1.f;
            rescale_o(alpha);
            l_part *= alpha;
            m_used = fmaxf(m_used, m_pend);
          }
          // recovery path: the stream's previous PV (o_prev), or also this stage's PV of the part
          // of P already handed over (o_lo), known complete
          bool o_prev = false, o_lo = false;
#pragma unroll
          for (int q = 0; q < kTile / 32; ++q) {
            uint32_t pw[16];
            float2 cs;
            chunk_exps(sr + 32 * q, q, m_used, pw, cs);
            const bool big = !(cs.x + cs.y <= 1.8446744e19f);  // 2^64, or inf / NaN
            if (__any_sync(0xffffffffu, big)) {
              // rare: raise this row's reference to the chunk's largest logit, rescale O_x, l,
              // this stage's sums and its P chunks already stored, then redo the chunk
              float xm = -INFINITY;
#pragma unroll
              for (int c = 0; c < 32; ++c)
                if (32 * q + c < valid) xm = fmaxf(xm, fmaf(__uint_as_float(sr[32 * q + c]), sl2, -m_used));
              // the raise is a whole number of octaves, so that rescaling bf16 P is exact
              const bool raise = big && xm > 0.f;
              const float xr = raise ? fminf(ceilf(xm), 1024.f) : 0.f;
              const int n = static_cast<int>(xr);
              const float alpha = n >= 127 ? 0.f : __int_as_float((127 - n) << 23);  // 2^-n
              // After the first part of P has been handed over (q >= kPSplit), its PV is waited
              // for and then rescaled inside O_x with everything before it; only the chunks stored
              // since are rescaled in place.  (A pending raise above already waited for the previous
              // PV: that wait then returns at once.)
              if (q >= kPSplit && !o_lo) {
                if (!mbar_wait_warp(pvlo_done + x, sc & 1, abort_flag, wl)) { ok = false; break; }
                tc_fence_after();
                o_lo = o_prev = true;
              } else if (!o_prev) {
                if (!mbar_wait_warp(pv_done + x, (sc - 1) & 1, abort_flag, wl)) { ok = false; break; }
                tc_fence_after();
                o_prev = true;
              }
              tmem_st_wait();
              rescale_o(alpha);
              l_part *= alpha;
              rs.x *= alpha;
              rs.y *= alpha;
#pragma unroll 1
              for (int q2 = q >= kPSplit ? kPSplit : 0; q2 < q; ++q2) {
                uint32_t pv[16];
                tmem_ld16(tS + 16 * q2, pv);
                tmem_ld_wait_regs16(pv);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pv[i]));
                  pv[i] = pack_bf16x2(f.x * alpha, f.y * alpha);
                }
                tmem_st16(tS + 16 * q2, pv);
              }
              tmem_st_wait();
              m_used += xr;
              chunk_exps(sr + 32 * q, q, m_used, pw, cs);
            }
            rs = __fadd2_rn(rs, cs);
            tmem_st16(tS + 16 * q, pw);
            if (q == kPSplit - 1) signal_half();
          }
          if (!ok) break;
          const float st = rs.x + rs.y;  // this stage's P sum against m_used
          m_pend = st > 65536.f ? m_used + __log2f(st) : -INFINITY;
        }
        l_part += rs.x + rs.y;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full + x);
      }
      if (!ok) break;
      if (SPARSE && live && static_cast<unsigned>(qrow) >= static_cast<unsigned>(p.N)) live = false;
      const size_t rbase = (static_cast<size_t>(bh) * p.N + qrow) * HD + x * (HD / 2);
      const bool store = live && (MODE != kDense || p.store_out);
      // the half row of R (reuse) or O_full (residual) this thread combines: its loads are in
      // flight while the stream's last PV completes and the two streams exchange (m, l)
      constexpr int NV = HD / 16;  // uint4 (8 bf16) per half row
      uint4 extra[MODE == kDense ? 1 : NV];
      if (MODE != kDense) {
        const __nv_bfloat16* src = MODE == kReuse ? p.R_in : p.O_full;
        const bool use = store && src != nullptr;
#pragma unroll
        for (int i = 0; i < NV; ++i)
          extra[i] = use ? *reinterpret_cast<const uint4*>(src + rbase + 8 * i) : make_uint4(0u, 0u, 0u, 0u);
      }
      const bool has_b = T > 1;  // stream B has at least one stage in this unit
      if (x == 0 || has_b) {
        // this stream's last PV of the unit
        if (!mbar_wait_warp(pv_done + x, (sc - 1) & 1, abort_flag, wl)) { ok = false; break; }
        tc_fence_after();
      }
      // both streams' (m, l) of each row: exchange through shared memory between two bounded
      // mbarrier rendezvous of the row group's two warps (written / read)
      sXch[x * kTile + row] = make_float2(m_used, l_part);
      tc_fence_before();  // (the partner's completed PVs are ordered before this warp's O reads)
      mbar_arrive(pair + rg);
      if (!mbar_wait_warp(pair + rg, 0, abort_flag, wl)) { ok = false; break; }
      tc_fence_after();
      const float2 xa = sXch[row], xb = sXch[kTile + row];
      mbar_arrive(pair + rg);
      if (!mbar_wait_warp(pair + rg, 1, abort_flag, wl)) { ok = false; break; }
      const float m_all = fmaxf(xa.x, xb.x);  // finite: stream A always holds a valid key
      const float wA = fast_exp2(xa.x - m_all);
      const float wB = has_b ? fast_exp2(xb.x - m_all) : 0.f;
      const float l_sum = xa.y * wA + xb.y * wB;
      // ---- epilogue: this thread's output row, columns [x*HD/2, (x+1)*HD/2); its half rows of
      // O_A and O_B in one TMEM round trip
      const float inv_l = 1.f / l_sum;
      const float cA = wA * inv_l, cB = wB * inv_l;
      const uint32_t tOA = tmem + lane_base + kTmO + x * (HD / 2), tOB = tOA + HD;
      uint32_t oab[HD];  // [0, HD/2): O_A; [HD/2, HD): O_B
      if constexpr (HD == 128) tmem_ld32x4_wait(tOA, tOA + 32, tOB, tOB + 32, oab);
      else tmem_ld32x2_wait(tOA, tOB, oab);
      if (store) {
#pragma unroll
        for (int c = 0; c < HD / 2; c += 8) {
          float v[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            // O_B holds no product of this unit when stream B had no stage: leave it out
            const float b = has_b ? __uint_as_float(oab[HD / 2 + c + i]) * cB : 0.f;
            v[i] = fmaf(__uint_as_float(oab[c + i]), cA, b);
          }
          if (MODE != kDense) {
            const uint4 rr = extra[c / 8];
            const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rr);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = __bfloat1622float2(r2[i]);
              if (MODE == kReuse) {  // O_hat = O_s + R (R = 0 when none is given)
                v[2 * i] += f.x;
                v[2 * i + 1] += f.y;
              } else {               // R = O_full - O_s
                v[2 * i] = f.x - v[2 * i];
                v[2 * i + 1] = f.y - v[2 * i + 1];
              }
            }
          }
          uint4 w;
          w.x = pack_bf16x2(v[0], v[1]);
          w.y = pack_bf16x2(v[2], v[3]);
          w.z = pack_bf16x2(v[4], v[5]);
          w.w = pack_bf16x2(v[6], v[7]);
          *reinterpret_cast<uint4*>(p.out + rbase + c) = w;
        }
      }
      if (MODE == kDense && x == 0 && live && p.lse != nullptr) {
        p.lse[static_cast<size_t>(bh) * p.N + qrow] = (m_all + __log2f(l_sum)) * 0.69314718055994531f;
      }
      tc_fence_before();
      mbar_arrive(o_empty);
    }
    // (after an abort) no load or store of this warp is still in flight when TMEM is released
    tmem_ld_wait();
    tmem_st_wait();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mcs
