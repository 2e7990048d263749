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
// N.  Eight scorer warps: warp w owns keys 32*(w%4) .. +31 of the tile (its TMEM lanes) and the
// query half w/4, and sums its half of each key's row in registers; the two half sums go to
// this CTA's slice of a global scratch buffer.  After the last tile the same warps add the
// halves (one fp32 addition, so the score does not depend on any ordering), run an exact radix
// select on the fp32 bit patterns (scores are non-negative, so bit order is value order) and
// an order-preserving compaction that emits the chosen keys in ascending order.  Warps 8-11
// copy the group's queries (gathered by perm) and the key tiles with cp.async; warp 12 issues
// the MMAs.
#pragma once

#include "sm100.cuh"

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
};

constexpr int kSelThreads = 416;
constexpr int kSelScorers = 256;

template <int HD>
struct SelectSmem {
  static constexpr int STAGES = 4;
  static constexpr uint32_t TILE_BYTES = 128 * HD * 2;
  static constexpr uint32_t Q_OFF = 0;
  static constexpr uint32_t K_OFF = TILE_BYTES;
  static constexpr uint32_t L_OFF = K_OFF + STAGES * TILE_BYTES;  // 128 floats
  static constexpr uint32_t HIST_OFF = L_OFF + 512;               // 256 ints
  static constexpr uint32_t SCAN_OFF = HIST_OFF + 1024;           // 32 ints
  static constexpr uint32_t BAR_OFF = SCAN_OFF + 128;
  // q_full, q_empty, k_full[S], k_empty[S], s_full[2], s_empty[2], drain, join
  static constexpr int NBAR = 2 + 2 * STAGES + 4 + 2;
  static constexpr uint32_t MISC_OFF = BAR_OFF + NBAR * 8;
  static constexpr uint32_t BYTES = MISC_OFF + 16;  // window is 1024-aligned (checked)
};

// Top-k of scores[0..N) by the 256 scorer threads (named barrier 1), given the two half sums
// a[] and b[]: the first radix pass stores a[j] + b[j] into a[]; writes k ascending indices.
__device__ __forceinline__ void topk_select_256(float* a, const float* b, int N, int k, int32_t* out, int* hist,
                                                int* scan) {
  constexpr int NT = kSelScorers, NW = NT / 32;
  const int t = threadIdx.x;
  const int w = t >> 5, l = t & 31;
  uint32_t* bits = reinterpret_cast<uint32_t*>(a);
  uint32_t prefix = 0, pmask = 0;
  int kk = k;
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    hist[t] = 0;
    named_sync(1, NT);
    if (pass == 0) {
      for (int j = t; j < N; j += NT) {
        const float sc = a[j] + b[j];
        a[j] = sc;
        atomicAdd(&hist[__float_as_uint(sc) >> 24], 1);
      }
    } else {
      for (int j = t; j < N; j += NT) {
        const uint32_t u = bits[j];
        if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
      }
    }
    named_sync(1, NT);
    if (w == 0) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      int h[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        h[i] = hist[255 - 8 * l - i];
        s += h[i];
      }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (l >= o) incl += v;
      }
      const int excl = incl - s;
      if (excl < kk && kk <= incl) {
        int above = excl;
        int digit = 255 - 8 * l;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above + h[i] >= kk) {
            digit = 255 - 8 * l - i;
            break;
          }
          above += h[i];
        }
        scan[0] = digit;
        scan[1] = above;
      }
    }
    named_sync(1, NT);
    const uint32_t digit = static_cast<uint32_t>(scan[0]);
    kk -= scan[1];
    prefix |= digit << shift;
    pmask |= 255u << shift;
  }
  // prefix = bit pattern of the k-th largest score; take all larger ones and the first kk
  // equal ones in index order.
  const uint32_t T = prefix;
  const int need_eq = kk;
  int out_pos = 0, eq_seen = 0;
  named_sync(1, NT);
#pragma unroll 1
  for (int base = 0; base < N; base += NT) {
    const int j = base + t;
    const bool valid = j < N;
    const uint32_t u = valid ? bits[j] : 0u;
    const bool gt = valid && u > T;
    const bool eq = valid && u == T;
    const uint32_t beq = __ballot_sync(0xffffffffu, eq);
    if (l == 0) scan[4 + w] = __popc(beq);
    named_sync(1, NT);
    int eq_before = eq_seen, eq_total = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      eq_before += i < w ? scan[4 + i] : 0;
      eq_total += scan[4 + i];
    }
    eq_before += __popc(beq & ((1u << l) - 1u));
    const bool take = gt || (eq && eq_before < need_eq);
    const uint32_t btk = __ballot_sync(0xffffffffu, take);
    if (l == 0) scan[16 + w] = __popc(btk);
    named_sync(1, NT);
    int pos = out_pos, tk_total = 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      pos += i < w ? scan[16 + i] : 0;
      tk_total += scan[16 + i];
    }
    pos += __popc(btk & ((1u << l) - 1u));
    if (take) out[pos] = j;
    out_pos += tk_total;
    eq_seen += eq_total;
    named_sync(1, NT);
  }
}

template <int HD, int CQ>
__global__ void __launch_bounds__(kSelThreads, 1)
    select_kernel(const __grid_constant__ CUtensorMap tmK, const SelectParams p) {
  using L = SelectSmem<HD>;
  constexpr int STAGES = L::STAGES;
  constexpr int CHUNKS = HD / 8;
  constexpr int ROWS_PER_IT = 32 / CHUNKS;
  constexpr uint32_t HALF = 128 * 128;
  constexpr uint32_t IDESC = idesc_bf16(128, 128, false, false);
  constexpr int QH = CQ / 2;  // query columns per scorer warp

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
  uint64_t* s_empty = s_full + 2;
  uint64_t* drain = s_empty + 2;
  uint64_t* join = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gptr + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gptr + L::MISC_OFF + 4);
  float* sL = reinterpret_cast<float*>(gptr + L::L_OFF);
  int* hist = reinterpret_cast<int*>(gptr + L::HIST_OFF);
  int* scan = reinterpret_cast<int*>(gptr + L::SCAN_OFF);
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full + b, 1);
      mbar_init(s_empty + b, kSelScorers);
    }
    mbar_init(drain, 1);
    mbar_init(join, kSelScorers);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 12) {
    tmem_alloc(tmem_slot, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int T = p.key_tiles;

  if (warp >= 8 && warp < 12) {
    // ------------------------------------------------------------------ producer
    const int pw = warp - 8;
    const int sub = lane / CHUNKS, c = lane % CHUNKS;
    uint32_t k_it = 0, u_it = 0;
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
      if (pw != 0) continue;  // warp 8 alone streams the key tiles, two 64-column TMA boxes each
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
        __syncwarp();
      }
      if (*abort_flag) break;
    }
    cp_async_wait_all();
  } else if (warp == 12) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // descriptors of stage 0 / of Q; stages and k-steps only move the start-address field
      const uint64_t dK0 = desc_sw128(sK, 16, 1024), dQ = desc_sw128(sQ, 16, 1024);
      constexpr uint64_t kStageStep = L::TILE_BYTES >> 4;
      uint32_t k_it = 0, s_it = 0, u_it = 0;
      bool ok = true;
      for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x, ++u_it) {
        ok = mbar_wait(q_full, u_it & 1, abort_flag);
        for (int j = 0; j < T && ok; ++j, ++k_it, ++s_it) {
          const uint32_t st = k_it % STAGES, b = s_it & 1;
          ok = mbar_wait(k_full + st, (k_it / STAGES) & 1, abort_flag) &&
               mbar_wait(s_empty + b, ((s_it >> 1) & 1) ^ 1, abort_flag);
          if (!ok) break;
          fence_proxy_async_smem();
          tc_fence_after();
          const uint64_t dK = dK0 + st * kStageStep;
#pragma unroll
          for (int ks = 0; ks < HD / 16; ++ks) {
            const uint64_t koff = (((ks >> 2) * HALF + (ks & 3) * 32) >> 4);
            mma_bf16_ss(tmem + b * 128, dK + koff, dQ + koff, IDESC, ks > 0 ? 1u : 0u);
          }
          mma_commit(k_empty + st);
          mma_commit(s_full + b);
          if (j == T - 1) mma_commit(q_empty);
        }
      }
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
    // ------------------------------------------------------------------ scorers + top-k
    const int t = threadIdx.x;  // 0..255
    const int rg = warp & 3, ch = warp >> 2;
    const uint32_t tS = tmem + (static_cast<uint32_t>(rg * 32) << 16) + ch * QH;
    const float sl2 = p.scale_log2;
    float* part0 = p.scratch + static_cast<size_t>(blockIdx.x) * 2 * p.scratch_stride;
    float* part1 = part0 + p.scratch_stride;
    float* mine = ch ? part1 : part0;
    uint32_t s_it = 0, jn = 0;
    bool ok = true;
    for (int unit = blockIdx.x; unit < p.num_units && ok; unit += gridDim.x) {
      const int bh = unit / p.G;
      const int g = unit - bh * p.G;
      const size_t head_off = static_cast<size_t>(bh) * p.N;
      if (t < CQ) {
        int q = p.perm[head_off + static_cast<size_t>(g) * CQ + t];
        if (static_cast<unsigned>(q) >= static_cast<unsigned>(p.N)) q = 0;
        sL[t] = p.lse[head_off + q] * 1.4426950408889634f;
      }
      mbar_arrive(join);
      if (!mbar_wait_rendezvous(join, (jn++) & 1, abort_flag)) { ok = false; break; }
      for (int j = 0; j < T; ++j, ++s_it) {
        const uint32_t b = s_it & 1;
        if (!mbar_wait_warp(s_full + b, (s_it >> 1) & 1, abort_flag)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[QH];
#pragma unroll
        for (int c = 0; c < QH; c += 32) tmem_ld32(tS + b * 128 + c, sr + c);
        tmem_ld_wait_regs(sr);
#pragma unroll
        for (int c = 32; c < QH; c += 32) reg_fence32(sr + c);
        tc_fence_before();
        mbar_arrive(s_empty + b);
        const float* lq = sL + ch * QH;
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int c = 0; c < QH; c += 4) {
          const float4 lv = *reinterpret_cast<const float4*>(lq + c);
          acc0 += fast_exp2(fmaf(__uint_as_float(sr[c + 0]), sl2, -lv.x));
          acc1 += fast_exp2(fmaf(__uint_as_float(sr[c + 1]), sl2, -lv.y));
          acc0 += fast_exp2(fmaf(__uint_as_float(sr[c + 2]), sl2, -lv.z));
          acc1 += fast_exp2(fmaf(__uint_as_float(sr[c + 3]), sl2, -lv.w));
        }
        const int key = j * 128 + rg * 32 + lane;
        if (key < p.N) mine[key] = acc0 + acc1;
      }
      if (!ok) break;
      // every scorer has stored its half sums before any of them reads the other half
      mbar_arrive(join);
      if (!mbar_wait_rendezvous(join, (jn++) & 1, abort_flag)) { ok = false; break; }
      topk_select_256(part0, part1, p.N, p.k, p.idx + (static_cast<size_t>(bh) * p.G + g) * p.k, hist, scan);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 12) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace mcs
