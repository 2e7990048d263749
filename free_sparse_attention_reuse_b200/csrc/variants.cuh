// The selection variants of the controlled oracle comparison, at equal attention density.
//
// "MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 어떻게 동작하나: a block oracle
// picks KV blocks per query block, a token oracle shares one selection of individual KV tokens
// per query block, a per-query oracle picks KV tokens for every query on its own, all three by
// exact dense attention probabilities; they are compared with vanilla block-sparse attention
// (BSA), which estimates block importance from mean-pooled query and key representations.
// Section 무엇인가: most block-sparse methods score blocks with mean-pooled queries and keys.
//
// Here:
//   * block oracle  — select_kernel in block mode (exact per-key group scores, summed per KV
//                      block of BK keys) followed by block_select_256 below;
//   * vanilla BSA   — bsa_pool_kernel (mean of each KV block's keys) and bsa_select_kernel
//                      (mean of the group's queries, pooled logit q̄·k̄ per block);
//   * token oracle  — the ordinary selection with contiguous query blocks (perm = identity);
//   * per-query     — perquery_attn_kernel: every query attends to its own k keys of largest
//                      logit (= largest probability), renormalised over that set.
// Block selections are emitted as token indices (kb whole blocks, ascending) so that the
// ordinary sparse attention kernel runs them unchanged.
#pragma once

#include "sm100.cuh"

namespace mcs {

// Pick the kb largest of the nb block scores s[] (shared memory), ties to the lower block, and
// write the token indices of the chosen blocks, ascending: out[i*BK + r] = b_i*BK + r.  Runs on
// the first NT threads of the block (named barrier `bar`); flag[] is shared scratch of nb ints
// and red[] of NT/32 + 1 ints.  O(nb^2 / NT) comparisons: nb is N / BK (at most a few thousand).
template <int NT>
__device__ __forceinline__ void block_select(const float* s, int nb, int kb, int BK, int32_t* out, int* flag,
                                             int* red, uint32_t bar) {
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  for (int b = t; b < nb; b += NT) {
    const float v = s[b];
    int rank = 0;
    for (int c = 0; c < nb; ++c) {
      const float u = s[c];
      rank += (u > v || (u == v && c < b)) ? 1 : 0;
    }
    flag[b] = rank < kb ? 1 : 0;
  }
  named_sync(bar, NT);
  // exclusive scan of the flags over contiguous per-thread ranges
  const int per = (nb + NT - 1) / NT;
  const int b0 = min(nb, t * per), b1 = min(nb, b0 + per);
  int cnt = 0;
  for (int b = b0; b < b1; ++b) cnt += flag[b];
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (l >= o) incl += v;
  }
  if (l == 31) red[w] = incl;
  named_sync(bar, NT);
  int base = incl - cnt;
  for (int i = 0; i < w; ++i) base += red[i];
  for (int b = b0; b < b1; ++b) {
    if (flag[b]) {
      int32_t* o = out + static_cast<size_t>(base) * BK;
      for (int r = 0; r < BK; ++r) o[r] = b * BK + r;
      ++base;
    }
  }
  named_sync(bar, NT);
}

// ---------------------------------------------------------------------------------- BSA
struct BsaParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const int32_t* perm;  // [BH, N]
  float* kbar;          // [BH, nb, d] mean of each KV block's keys
  int32_t* idx;         // [BH, G, kb*BK]
  int BH, N, C, G, d, BK, nb, kb;
};

// kbar[bh, b, :] = mean of keys b*BK .. b*BK+BK-1 (fp32).  grid (nb, BH), blockDim = d.
__global__ void bsa_pool_kernel(const BsaParams p) {
  const int b = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  if (c >= p.d) return;
  const __nv_bfloat16* Kb = p.K + (static_cast<size_t>(bh) * p.N + static_cast<size_t>(b) * p.BK) * p.d + c;
  float acc = 0.f;
  for (int r = 0; r < p.BK; ++r) acc += __bfloat162float(Kb[static_cast<size_t>(r) * p.d]);
  p.kbar[(static_cast<size_t>(bh) * p.nb + b) * p.d + c] = acc / static_cast<float>(p.BK);
}

constexpr int kBsaThreads = 256;

// One group per block: q̄ = mean of its queries, pooled logit q̄·k̄_b per KV block, kb largest.
// grid (G, BH), 256 threads, dynamic shared memory (d + 2*nb + 16) * 4 bytes.
__global__ void __launch_bounds__(kBsaThreads) bsa_select_kernel(const BsaParams p) {
  extern __shared__ __align__(16) float bsm[];
  float* qbar = bsm;
  float* sc = qbar + p.d;
  int* flag = reinterpret_cast<int*>(sc + p.nb);
  int* red = flag + p.nb;
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int32_t* members = p.perm + static_cast<size_t>(bh) * p.N + static_cast<size_t>(g) * p.C;
  const __nv_bfloat16* Qh = p.Q + static_cast<size_t>(bh) * p.N * p.d;
  if (t < p.d) {
    float acc = 0.f;
    for (int r = 0; r < p.C; ++r) {
      int q = members[r];
      if (static_cast<unsigned>(q) >= static_cast<unsigned>(p.N)) {
        raise_status(kStatusBadIndex);
        q = 0;
      }
      acc += __bfloat162float(Qh[static_cast<size_t>(q) * p.d + t]);
    }
    qbar[t] = acc / static_cast<float>(p.C);
  }
  __syncthreads();
  const float* kb = p.kbar + static_cast<size_t>(bh) * p.nb * p.d;
  for (int b = t; b < p.nb; b += kBsaThreads) {
    float acc = 0.f;
    for (int c = 0; c < p.d; ++c) acc = fmaf(qbar[c], kb[static_cast<size_t>(b) * p.d + c], acc);
    sc[b] = acc;
  }
  __syncthreads();
  block_select<kBsaThreads>(sc, p.nb, p.kb, p.BK, p.idx + (static_cast<size_t>(bh) * p.G + g) * p.kb * p.BK, flag,
                            red, 1);
}

// ---------------------------------------------------------------------------------- per-query
struct PerQueryParams {
  const __nv_bfloat16* Q;
  const __nv_bfloat16* K;
  const __nv_bfloat16* V;
  __nv_bfloat16* out;
  float* scratch;  // gridDim.x * kPqWarps slices of N floats (the logits of one query each)
  int BH, N, d, k;
  float scale;
  long long num_rows;  // BH * N
};

constexpr int kPqWarps = 16;
constexpr int kPqKeys = 32;  // keys per shared-memory tile

// Orderable 32-bit key of a float: unsigned order = float order.
__device__ __forceinline__ uint32_t f2key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Persistent CTAs of 16 warps; each pass takes 16 consecutive query rows of one head (warp w:
// row 16*i + w).  Phase 1: the 16 queries' logits over all keys, key tiles staged in shared
// memory and shared by the warps, into the warp's scratch row.  Phase 2: the k-th largest logit
// by a 4-pass radix select on orderable keys (warp-private 256-bin histograms).  Phase 3: the
// softmax over the chosen keys (every key above the threshold, and the first keys equal to it
// in key order) and the weighted sum of their values.  CUDA cores only: this is the analysis
// variant, O(N^2 d) work per head.
template <int HD>
__global__ void __launch_bounds__(kPqWarps * 32, 1) perquery_attn_kernel(const PerQueryParams p) {
  constexpr int KS = HD + 1;  // padded row stride (floats) of the key tile: lanes hit distinct banks
  __shared__ float sQ[kPqWarps][HD];
  __shared__ float sK[kPqKeys][KS];
  __shared__ int sHist[kPqWarps][256];
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  float* lg = p.scratch + (static_cast<size_t>(blockIdx.x) * kPqWarps + w) * p.N;
  const long long batches = (p.num_rows + kPqWarps - 1) / kPqWarps;
  for (long long bt = blockIdx.x; bt < batches; bt += gridDim.x) {
    const long long row0 = bt * kPqWarps;  // rows never straddle heads: N is a multiple of 16
    const long long row = row0 + w;
    const bool live = row < p.num_rows;
    const size_t head = static_cast<size_t>(row0 / p.N);
    const __nv_bfloat16* Kh = p.K + head * p.N * HD;
    const __nv_bfloat16* Vh = p.V + head * p.N * HD;
    for (int c = l; c < HD; c += 32)
      sQ[w][c] = live ? __bfloat162float(p.Q[static_cast<size_t>(row) * HD + c]) * p.scale : 0.f;
    // phase 1: logits
    for (int j0 = 0; j0 < p.N; j0 += kPqKeys) {
      __syncthreads();
      for (int e = threadIdx.x; e < kPqKeys * HD; e += kPqWarps * 32) {
        const int r = e / HD, c = e - r * HD;
        const int j = j0 + r;
        sK[r][c] = j < p.N ? __bfloat162float(Kh[static_cast<size_t>(j) * HD + c]) : 0.f;
      }
      __syncthreads();
      const int j = j0 + l;
      float acc = 0.f;
#pragma unroll 8
      for (int c = 0; c < HD; ++c) acc = fmaf(sQ[w][c], sK[l][c], acc);
      if (j < p.N) lg[j] = acc;
    }
    __syncwarp();
    if (!live) continue;
    // phase 2: the k-th largest logit (ties resolved below, lower key first)
    uint32_t prefix = 0, pmask = 0;
    int kk = p.k;
    for (int pass = 0; pass < 4; ++pass) {
      const int shift = 24 - 8 * pass;
      for (int i = l; i < 256; i += 32) sHist[w][i] = 0;
      __syncwarp();
      for (int j = l; j < p.N; j += 32) {
        const uint32_t u = f2key(lg[j]);
        if ((u & pmask) == prefix) atomicAdd(&sHist[w][(u >> shift) & 255u], 1);
      }
      __syncwarp();
      // lane l owns digits 255-8l .. 248-8l (descending)
      int h[8], sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        h[i] = sHist[w][255 - 8 * l - i];
        sum += h[i];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (l >= o) incl += v;
      }
      const int excl = incl - sum;
      int digit = 0, above = 0;
      const bool mine = excl < kk && kk <= incl;
      if (mine) {
        above = excl;
        digit = 255 - 8 * l;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (above + h[i] >= kk) {
            digit = 255 - 8 * l - i;
            break;
          }
          above += h[i];
        }
      }
      const uint32_t who = __ballot_sync(0xffffffffu, mine);
      const int src = who ? __ffs(who) - 1 : 0;  // exactly one lane holds the k-th key's digit
      digit = __shfl_sync(0xffffffffu, digit, src);
      above = __shfl_sync(0xffffffffu, above, src);
      prefix |= static_cast<uint32_t>(digit) << shift;
      pmask |= 255u << shift;
      kk -= above;
      __syncwarp();
    }
    const uint32_t T = prefix;  // orderable key of the k-th largest logit
    const int need_eq = kk;     // keys equal to it that are taken, lowest index first
    // phase 3: softmax over the chosen keys; the row max is the largest logit
    float mx = -INFINITY;
    for (int j = l; j < p.N; j += 32) mx = fmaxf(mx, lg[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    constexpr int PER = HD / 32;  // output columns per lane
    float o[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) o[i] = 0.f;
    float lsum = 0.f;
    int eq_seen = 0;
    for (int j0 = 0; j0 < p.N; j0 += 32) {
      const int j = j0 + l;
      const float x = j < p.N ? lg[j] : -INFINITY;
      const uint32_t u = j < p.N ? f2key(x) : 0u;
      const bool eq = j < p.N && u == T;
      const uint32_t beq = __ballot_sync(0xffffffffu, eq);
      const bool take = (j < p.N && u > T) || (eq && eq_seen + __popc(beq & ((1u << l) - 1u)) < need_eq);
      eq_seen += __popc(beq);
      uint32_t bt2 = __ballot_sync(0xffffffffu, take);
      const float wj = take ? __expf(x - mx) : 0.f;
      lsum += wj;
      while (bt2) {  // the warp walks the chosen keys of this chunk, lanes split the columns
        const int src = __ffs(bt2) - 1;
        bt2 &= bt2 - 1;
        const float wv = __shfl_sync(0xffffffffu, wj, src);
        const __nv_bfloat16* vr = Vh + static_cast<size_t>(j0 + src) * HD;
#pragma unroll
        for (int i = 0; i < PER; ++i) o[i] = fmaf(wv, __bfloat162float(vr[l + 32 * i]), o[i]);
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    const float inv = 1.f / lsum;
#pragma unroll
    for (int i = 0; i < PER; ++i) p.out[static_cast<size_t>(row) * HD + l + 32 * i] = __float2bfloat16(o[i] * inv);
  }
}

}  // namespace mcs
