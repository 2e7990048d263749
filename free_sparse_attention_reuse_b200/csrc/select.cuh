// Exact selection, pass 2: group scores from exact softmax probabilities, then top-k.
//
// "MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 어떻게 쓰나: an online-softmax
// kernel exposes no logits, so selection runs in two passes; pass 1 is the per-query
// log-sum-exp (emitted by the dense kernel), pass 2 recomputes the logits and turns them into
// exact probabilities.  Section 어떻게 동작하나: the token oracle shares one selection per
// query block and picks individual KV tokens by exact dense probabilities.
//
// For group g (queries perm[g*C .. g*C+C-1]) and every key j:
//     score_g[j] = sum_{i in g} exp2(scale*log2(e) * q_i.k_j - LSE_i*log2(e))
// and idx[g, :] = the k keys of largest score, ties to the lower key index, ascending.
//
// One CTA per SM, persistent over groups.  The logits are computed transposed on tcgen05:
// S^T = K_tile Q_g^T with the 128 keys of a tile on M (TMEM lanes) and the group's queries on
// N, in four TMEM buffers.  Sixteen scorer warps in four quarters take every fourth tile (tile
// s lands in buffer s % 4 and is scored by quarter s % 4), so that four warps of each SM
// sub-partition keep the exponential unit busy; within a quarter, warp w owns keys
// 32*(w%4) .. +31 of the tile (its TMEM lanes) and sums the row of each key in registers (two
// 64-column TMEM loads), stores the score to this CTA's slice of a global scratch buffer and
// counts it in a shared-memory histogram of its top bits.  After the last tile, scorer warps
// 0-7 run an exact radix select on the fp32 bit patterns (scores are non-negative, so bit
// order is value order): the keys in the threshold bin go to a candidate list in shared memory,
// where the remaining bits are resolved, and an order-preserving compaction emits the chosen
// keys in ascending order.  Warps 16-19 gather the group's queries (by perm) with cp.async;
// warp 16 streams the key tiles by TMA; warp 20 issues the MMAs.
#pragma once

#include "sm100.cuh"
#include "variants.cuh"

namespace mcs {

struct SelectParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const int32_t* perm;   // [BH, N]
  const float* lse;      // [BH, N] natural log
  int32_t* idx;          // [BH, G, k]
  float* scratch;        // gridDim.x slices of 2 * scratch_stride floats
  size_t scratch_stride;
  int BH, N, C, G, k;
  int key_tiles;         // ceil(N / 128)
  int num_units;         // BH * G
  float scale_log2;
  int BK, kb;            // block mode (BK > 0): the kb KV blocks of BK keys with the largest
                         // summed score, emitted as k = kb*BK token indices
};

// Six warpgroups: scorers (warps 0-15), producers (16-19), MMA issuer (warp 20; 21-23 complete
// the warpgroup).  768 threads are launched with 80 registers each (65536 / 768 rounded down to
// the allocation granularity of 8); setmaxnreg splits those 61440 registers 96 (four scorer
// warpgroups) / 56 / 40 per thread.
constexpr int kSelThreads = 768;
constexpr uint32_t kSelLaunchRegs = (65536 / kSelThreads) & ~7u;  // 80 (checked on the host)
constexpr uint32_t kSelRegsScorer = 96, kSelRegsProducer = 56, kSelRegsMma = 40;
static_assert(4 * 128 * kSelRegsScorer + 128 * kSelRegsProducer + 128 * kSelRegsMma <= kSelThreads * kSelLaunchRegs,
              "warpgroup register split exceeds the launch's registers");
constexpr int kSelScorerWarps = 16;
constexpr int kSelScorers = 256;  // threads of the top-k (scorer warps 0-7)
constexpr int kTopkBins = 4096;  // 12-bit radix digits
constexpr int kTopkCap = 4096;   // candidate list (shared memory) capacity

template <int HD>
struct SelectSmem {
  static constexpr int STAGES = 4;
  static constexpr uint32_t TILE_BYTES = 128 * HD * 2;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = TILE_BYTES;
  static constexpr uint32_t L_OFF = K_OFF + STAGES * TILE_BYTES;  // 128 floats
  static constexpr uint32_t HIST_OFF = L_OFF + 512;               // kTopkBins ints
  static constexpr uint32_t SCAN_OFF = HIST_OFF + kTopkBins * 4;  // 64 ints
  static constexpr uint32_t CAND_OFF = SCAN_OFF + 256;            // kTopkCap (bits, key) pairs
  static constexpr uint32_t BAR_OFF = CAND_OFF + kTopkCap * 8;
  // q_full, q_empty, k_full[S], k_empty[S], s_full[4], s_empty[4], drain, join
  static constexpr int NBAR = 2 + 2 * STAGES + 8 + 2;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr uint32_t BYTES = MISC_OFF + 16;  // window is 1024-aligned (checked)
  static_assert(BYTES + 1024 <= 227 * 1024, "selection tiles exceed the shared memory of one CTA");
};

// ---------------------------------------------------------------- exact top-k
//
// Radix select on the fp32 bit patterns of the scores (non-negative, so bit 31 is 0 and the
// order of the patterns is the order of the values), by three digits: bits 30-19, 18-7, 6-0.
// The histogram of the first digit is built while the scores are computed.  The key range is
// cut into eight contiguous chunks, one per scorer warp, so that a compaction by chunks emits
// ascending keys.  Scan slots: [0] digit, [1] count above it, [2] count in it, [3] candidate
// counter, [8+w] warp partial sums, [16+w] keys of chunk w above the prefix, [24+w] candidates
// of chunk w above the threshold, [32+w] keys of chunk w equal to the threshold.

// Find the bin of the kk-th largest element of hist[0..kTopkBins) (kk >= 1 and at most the
// total).  Thread t owns bins 4095-16t down to 4080-16t.
__device__ __forceinline__ void topk_find_bin(const int* hist, int kk, int* scan) {
  constexpr int NT = kSelScorers, NW = NT / 32, PER = kTopkBins / NT;
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  const int top = kTopkBins - 1 - PER * t;
  int h[PER], sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    h[i] = hist[top - i];
    sum += h[i];
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += v;
  }
  if (l == 31) scan[8 + w] = incl;
  named_sync(1, NT);
  int before = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) before += i < w ? scan[8 + i] : 0;
  incl += before;
  const int excl = incl - sum;
  if (excl < kk && kk <= incl) {
    int above = excl;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (above + h[i] >= kk) {
        scan[0] = top - i;
        scan[1] = above;
        scan[2] = h[i];
        break;
      }
      above += h[i];
    }
  }
  named_sync(1, NT);
}

__device__ __forceinline__ void topk_zero_hist(int* hist) {
  int4* h4 = reinterpret_cast<int4*>(hist);
  for (int i = threadIdx.x; i < kTopkBins / 4; i += kSelScorers) h4[i] = make_int4(0, 0, 0, 0);
}

// Shift and mask of the digit after the one at `shift` (19 -> 7 -> 0).
__device__ __forceinline__ int topk_next_shift(int shift) { return shift == 19 ? 7 : 0; }
__device__ __forceinline__ uint32_t topk_digit_mask(int shift) { return shift == 0 ? 127u : 4095u; }

// Top-k of score[0..N) by the 256 scorer threads (named barrier 1).  On entry hist holds the
// histogram of bits 30-19 of all N scores; writes k ascending key indices to out.
__device__ __forceinline__ void topk_select_256(const float* score, int N, int k, int32_t* out, int* hist,
                                                int* scan, uint2* cand) {
  constexpr int NT = kSelScorers, NW = NT / 32;
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  const uint32_t* bits = reinterpret_cast<const uint32_t*>(score);
  const uint32_t lt_mask = (1u << l) - 1u;
  int shift = 19;
  uint32_t prefix = 0, pmask = 0;
  int kk = k, cnt = N;
  // 1. digits over the whole key range, until the keys sharing the prefix fit the list
#pragma unroll 1
  for (;;) {
    topk_find_bin(hist, kk, scan);
    const uint32_t dm = topk_digit_mask(shift);
    prefix |= static_cast<uint32_t>(scan[0]) << shift;
    pmask |= dm << shift;
    kk -= scan[1];
    cnt = scan[2];
    if (cnt <= kTopkCap || shift == 0) break;
    topk_zero_hist(hist);
    named_sync(1, NT);
    shift = topk_next_shift(shift);
    const uint32_t nm = topk_digit_mask(shift);
    for (int j = t; j < N; j += NT) {
      const uint32_t u = bits[j];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & nm], 1);
    }
    named_sync(1, NT);
  }
  // 2. one pass over the chunks: count keys above the prefix, collect those sharing it
  const int chunk = ((N + NW - 1) / NW + 31) & ~31;
  const int j0 = min(N, w * chunk), j1 = min(N, j0 + chunk);
  if (t == 0) scan[3] = 0;
  if (t < NW) {
    scan[24 + t] = 0;
    scan[32 + t] = 0;
  }
  named_sync(1, NT);
  {
    int gt = 0, eq = 0;
    for (int jb = j0; jb < j1; jb += 256) {
      uint32_t u[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int j = jb + 32 * r + l;
        u[r] = j < j1 ? bits[j] : 0u;
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int j = jb + 32 * r + l;
        if (j < j1) {
          const uint32_t m = u[r] & pmask;
          if (m > prefix) {
            ++gt;
          } else if (m == prefix) {
            if (shift == 0) {
              ++eq;
            } else {
              const int pos = atomicAdd(&scan[3], 1);
              if (pos < kTopkCap) cand[pos] = make_uint2(u[r], static_cast<uint32_t>(j));
              else raise_status(kStatusBadShape);  // the histogram promised at most cnt keys
            }
          }
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      gt += __shfl_xor_sync(0xffffffffu, gt, o);
      eq += __shfl_xor_sync(0xffffffffu, eq, o);
    }
    if (l == 0) {
      scan[16 + w] = gt;
      if (shift == 0) scan[32 + w] = eq;
    }
  }
  named_sync(1, NT);
  // 3. the remaining digits over the candidate list; then per-chunk counts of its keys
  if (shift != 0) {
#pragma unroll 1
    while (shift != 0) {
      topk_zero_hist(hist);
      named_sync(1, NT);
      shift = topk_next_shift(shift);
      const uint32_t nm = topk_digit_mask(shift);
      for (int i = t; i < cnt; i += NT) {
        const uint32_t u = cand[i].x;
        if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & nm], 1);
      }
      named_sync(1, NT);
      topk_find_bin(hist, kk, scan);
      prefix |= static_cast<uint32_t>(scan[0]) << shift;
      pmask |= nm << shift;
      kk -= scan[1];
    }
    for (int i = t; i < cnt; i += NT) {
      const uint2 c = cand[i];
      const int wc = static_cast<int>(c.y) / chunk;
      if (c.x > prefix) atomicAdd(&scan[24 + wc], 1);
      else if (c.x == prefix) atomicAdd(&scan[32 + wc], 1);
    }
    named_sync(1, NT);
  }
  // 4. prefix = bit pattern T of the k-th largest score: take every key above it and the first
  // kk keys equal to it in key order, chunk by chunk.
  const uint32_t T = prefix;
  const int need_eq = kk;
  int out_base = 0, eq_seen = 0;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    if (i < w) {
      const int eqi = scan[32 + i];
      out_base += scan[16 + i] + scan[24 + i] + min(eqi, max(0, need_eq - eq_seen));
      eq_seen += eqi;
    }
  }
  for (int jb = j0; jb < j1; jb += 256) {
    uint32_t u[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = jb + 32 * r + l;
      u[r] = j < j1 ? bits[j] : 0u;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int j = jb + 32 * r + l;
      const bool in = j < j1;
      const bool eq = in && u[r] == T;
      const uint32_t beq = __ballot_sync(0xffffffffu, eq);
      const bool take = (in && u[r] > T) || (eq && eq_seen + __popc(beq & lt_mask) < need_eq);
      const uint32_t btk = __ballot_sync(0xffffffffu, take);
      if (take) out[out_base + __popc(btk & lt_mask)] = j;
      out_base += __popc(btk);
      eq_seen += __popc(beq);
    }
  }
}

template <int HD, int CQ, bool BLOCKS = false>
__global__ void __launch_bounds__(kSelThreads, 1)
    select_kernel(const __grid_constant__ CUtensorMap tmK, const SelectParams p) {
  using L = SelectSmem<HD>;
  constexpr int STAGES = L::STAGES;
  constexpr int CHUNKS = HD / 8;
  constexpr int ROWS_PER_IT = 32 / CHUNKS;
  constexpr uint32_t HALF = 128 * 128;
  constexpr uint32_t IDESC = idesc_bf16(128, 128, false, false);

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {
    if (threadIdx.x == 0) raise_status(kStatusBadShape);
    return;
  }
  uint8_t* gptr = smem_raw;
  uint64_t* bars = reinterpret_cast<uint64_t*>(gptr + L::BAR_OFF);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + STAGES;
  uint64_t* s_full = k_empty + STAGES;
  uint64_t* s_empty = s_full + 4;
  uint64_t* drain = s_empty + 4;
  uint64_t* join = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gptr + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gptr + L::MISC_OFF + 4);
  float* sL = reinterpret_cast<float*>(gptr + L::L_OFF);
  int* hist = reinterpret_cast<int*>(gptr + L::HIST_OFF);
  int* scan = reinterpret_cast<int*>(gptr + L::SCAN_OFF);
  uint2* cand = reinterpret_cast<uint2*>(gptr + L::CAND_OFF);
  const uint32_t sQ = base + L::Q_OFF;
  const uint32_t sK = base + L::K_OFF;
  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 128);
    mbar_init(q_empty, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(k_full + s, 1);  // one arrival with the expected bytes; the TMA completes them
      mbar_init(k_empty + s, 1);
    }
    for (int b = 0; b < 4; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, 128);  // buffer b: the 128 threads of scorer quarter b
    }
    mbar_init(drain, 1);
    mbar_init(join, kSelScorerWarps * 32);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 20) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int T = p.key_tiles;

  if (warp >= 16 && warp < 20) {
    // ------------------------------------------------------------------ producer
    regs_to<kSelRegsProducer, kSelLaunchRegs>();
    const int pw = warp - 16;
    const int sub = lane / CHUNKS, c = lane % CHUNKS;
    uint32_t k_it = 0, u_it = 0, k_issued = 0;
    for (int unit = blockIdx.x; unit < p.num_units; unit += gridDim.x, ++u_it) {
      const int bh = unit / p.G;
      const int g = unit - bh * p.G;
      const size_t head_off = static_cast<size_t>(bh) * p.N;
      const int my_row = pw * 32 + lane;
      int qi = my_row < CQ ? p.perm[head_off + static_cast<size_t>(g) * CQ + my_row] : -1;
      if (qi != -1 && static_cast<unsigned>(qi) >= static_cast<unsigned>(p.N)) {
        raise_status(kStatusBadIndex);
        qi = -1;
      }
      if (!mbar_wait(q_empty, (u_it & 1) ^ 1, abort_flag)) break;
#pragma unroll 4
      for (int it = 0; it < 32 / ROWS_PER_IT; ++it) {
        const int rl = it * ROWS_PER_IT + sub;
        const int q = __shfl_sync(0xffffffffu, qi, rl);
        const bool ok = q >= 0;
        cp_async16(sQ + sw128_offset(pw * 32 + rl, c, 128), p.Q + ((head_off + (ok ? q : 0)) * HD + c * 8),
                   ok ? 16u : 0u);
      }
      cp_async_arrive(q_full);
      if (pw != 0) continue;  // warp 16 alone streams the key tiles, two 64-column TMA boxes each
      for (int j = 0; j < T; ++j, ++k_it) {
        const uint32_t st = k_it % STAGES;
        if (!mbar_wait_warp(k_empty + st, ((k_it / STAGES) & 1) ^ 1, abort_flag)) break;
        if (lane == 0) {
          const uint32_t dst = sK + st * L::TILE_BYTES;
          mbar_arrive_expect_tx(k_full + st, L::TILE_BYTES);
#pragma unroll
          for (int h = 0; h < HD / 64; ++h)
            tma_load_2d(dst + h * HALF, &tmK, h * 64, static_cast<int>(head_off) + j * 128, k_full + st);
        }
        ++k_issued;
        __syncwarp();
      }
      if (*abort_flag) break;
    }
    cp_async_wait_all();
    if (pw == 0 && *abort_flag) {
      // after an abort, the key tiles already requested land before the CTA releases its
      // shared memory (the last load into each stage completes the phase counted for it)
      for (uint32_t s = 0; s < static_cast<uint32_t>(STAGES) && s < k_issued; ++s) {
        const uint32_t last = k_issued - 1 - ((k_issued - 1 + STAGES - s) % STAGES);
        mbar_drain(k_full + s, (last / STAGES) & 1);
      }
    }
  } else if (warp >= 20) {
    regs_to<kSelRegsMma, kSelLaunchRegs>();
    if (warp == 20) {
      // ------------------------------------------------------------------ MMA issuer
      // The whole warp runs the loop (its waits agree warp-wide); lane 0 issues each tcgen05
      // instruction, so the descriptors and counters are warp-uniform values.
      // descriptors of stage 0 / of Q; stages and k-steps only move the start-address field
      const uint64_t dK0 = desc_sw128(sK, 16, 1024), dQ = desc_sw128(sQ, 16, 1024);
      constexpr uint64_t kStageStep = L::TILE_BYTES >> 4;
      uint32_t k_it = 0, s_it = 0, u_it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x, ++u_it) {
        ok = mbar_wait_warp(q_full, u_it & 1, abort_flag);
        for (int j = 0; j < T && ok; ++j, ++k_it, ++s_it) {
          const uint32_t st = k_it % STAGES, b = s_it & 3;
          ok = mbar_wait_warp(k_full + st, (k_it / STAGES) & 1, abort_flag) &&
               mbar_wait_warp(s_empty + b, ((s_it >> 2) & 1) ^ 1, abort_flag);
          if (!ok) break;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t dK = dK0 + st * kStageStep;
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks) {
            const uint64_t koff = (((ks >> 2) * HALF + (ks & 3) * 32) >> 4);
            mma_bf16_ss_warp(tmem + b * 128, dK + koff, dQ + koff, IDESC, ks > 0 ? 1u : 0u);
          }
          mma_commit_warp(k_empty + st);
          mma_commit_warp(s_full + b);
          if (j == T - 1) mma_commit_warp(q_empty);
        }
      }
      mma_commit_warp(drain);
      mbar_drain(drain, 0);
    }  // warps 21-23 only complete the warpgroup
  } else {
    // ------------------------------------------------------------------ scorers + top-k
    regs_to<kSelRegsScorer, kSelLaunchRegs>();
    // S tile s (counted over the whole launch) lands in TMEM buffer s % 4 and is scored by
    // scorer quarter s % 4 (warps 4q .. 4q+3): each thread sums all CQ columns of its key.
    const int t = threadIdx.x;  // 0..511
    const int rg = warp & 3, quarter = warp >> 2;
    const bool topk_warp = warp < 8;  // warps 0-7 also run the top-k
    const uint32_t tS = tmem + (static_cast<uint32_t>(rg * 32) << 16);
    const float sl2 = p.scale_log2;
    float* score = p.scratch + static_cast<size_t>(blockIdx.x) * 2 * p.scratch_stride;
    uint32_t s0 = 0, jn = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x, s0 += T) {
      const int bh = unit / p.G;
      const int g = unit - bh * p.G;
      const size_t head_off = static_cast<size_t>(bh) * p.N;
      if (t < CQ) {
        int q = p.perm[head_off + static_cast<size_t>(g) * CQ + t];
        if (static_cast<unsigned>(q) >= static_cast<unsigned>(p.N)) q = 0;
        sL[t] = p.lse[head_off + q] * 1.4426950408889634f;
      }
      if (topk_warp) topk_zero_hist(hist);
      mbar_arrive(join);
      if (!mbar_wait_rendezvous(join, (jn++) & 1, abort_flag)) { ok = false; break; }
      for (int j = (quarter - static_cast<int>(s0)) & 3; j < T; j += 4) {
        const uint32_t sidx = s0 + j, b = sidx & 3;
        if (!mbar_wait_warp(s_full + b, (sidx >> 2) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        // the row's CQ columns, 64 at a time (the second load after the first half is summed);
        // the buffer is free for the next tile's MMA once both are in registers.  acc.x sums
        // the even columns and acc.y the odd ones (fp32 pairs: one packed instruction for two
        // columns), in column order.  One pair of columns in four takes its exponentials on the
        // FMA pipe (exp2_fma2, within the exponential unit's error), beside the exponential
        // unit's three.
        float2 acc = make_float2(0.f, 0.f);
        auto sum64 = [&](const uint32_t* sr, int c0) {
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float2 lv = *reinterpret_cast<const float2*>(sL + c0 + c);
            const float2 xv = __ffma2_rn(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                         make_float2(sl2, sl2), make_float2(-lv.x, -lv.y));
            const float2 e = (c / 2) % 4 == 3 ? exp2_fma2(xv) : make_float2(fast_exp2(xv.x), fast_exp2(xv.y));
            acc = __fadd2_rn(acc, e);
          }
        };
        uint32_t sr[64];
        tmem_ld64_wait(tS + b * 128, sr);
        if constexpr (CQ == 128) {
          sum64(sr, 0);
          tmem_ld64_wait(tS + b * 128 + 64, sr);
        }
        tc_fence_before();
        mbar_arrive(s_empty + b);
        sum64(sr, CQ - 64);
        const int key = j * 128 + rg * 32 + lane;
        if (key < p.N) {
          const float sc = acc.x + acc.y;
          score[key] = sc;
          atomicAdd(&hist[(__float_as_uint(sc) >> 19) & (kTopkBins - 1)], 1);
        }
      }
      if (!ok) break;
      // every score and histogram count is in place before the selection reads them
      mbar_arrive(join);
      if (!mbar_wait_rendezvous(join, (jn++) & 1, abort_flag)) { ok = false; break; }
      if (!topk_warp) continue;  // warps 8-15 wait for the next group at its first rendezvous
      int32_t* out = p.idx + (static_cast<size_t>(bh) * p.G + g) * p.k;
      if constexpr (BLOCKS) {
        // block oracle: exact probability mass of each KV block, then its kb largest
        float* blk = reinterpret_cast<float*>(cand);
        const int nb = p.N / p.BK;
        for (int b = t; b < nb; b += kSelScorers) {
          const float* sb = score + static_cast<size_t>(b) * p.BK;
          float acc = 0.f;
          for (int r = 0; r < p.BK; ++r) acc += sb[r];
          blk[b] = acc;
        }
        named_sync(1, kSelScorers);
        block_select<kSelScorers>(blk, nb, p.kb, p.BK, out, hist, scan, 1);
      } else {
        topk_select_256(score, p.N, p.k, out, hist, scan, cand);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 20) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mcs
