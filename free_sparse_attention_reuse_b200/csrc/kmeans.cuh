// Grouping-cost baseline: equal-size query groups from Lloyd's k-means, set against Fast PDDP
// ("MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 전제와 한계 compares the
// grouping cost of Fast PDDP with a k-means clustering; the pages give no algorithm for an
// equal-size k-means, so the one here is a reading, identical to the fp64 oracle's):
//   * G = N / C centroids, initialised as the means of the contiguous query blocks;
//   * `iters` Lloyd steps: every query goes to its nearest centroid (squared Euclidean distance
//     summed over the coordinates in order, each term rounded before it is added; ties to the
//     lower centroid), then every centroid becomes the mean of its queries (summed in query
//     order; an empty cluster keeps its centroid);
//   * equal sizes: clusters 0, 1, ..., G-1 in turn take the C not yet taken queries nearest to
//     their final centroid (ties to the lower query index).
// All arithmetic is fp64 in the oracle's order (no fused multiply-adds), so the groups match
// the oracle bit for bit.  This is a baseline for timing, not part of the hot path.
#pragma once

#include "sm100.cuh"

namespace mcs {

struct KmeansParams {
  const __nv_bfloat16* Q;  // [BH, N, d]
  double* cent;            // [BH, G, d]
  int32_t* assign;         // [BH, N]
  double* dist;            // [BH, G, N]  final distances, centroid-major
  unsigned char* taken;    // [BH, N]
  int32_t* perm;           // [BH, N]
  int BH, N, C, G, d;
};

__device__ __forceinline__ double km_bf2d(__nv_bfloat16 x) { return static_cast<double>(__bfloat162float(x)); }

// Initial centroids: the mean of block g's C rows.  grid (G, BH), block d threads.
__global__ void kmeans_init_kernel(const KmeansParams p) {
  const int g = blockIdx.x, bh = blockIdx.y, c = threadIdx.x;
  if (c >= p.d) return;
  const __nv_bfloat16* Qh = p.Q + static_cast<size_t>(bh) * p.N * p.d;
  double acc = 0.0;
  for (int i = g * p.C; i < (g + 1) * p.C; ++i) acc = __dadd_rn(acc, km_bf2d(Qh[static_cast<size_t>(i) * p.d + c]));
  p.cent[(static_cast<size_t>(bh) * p.G + g) * p.d + c] = __ddiv_rn(acc, static_cast<double>(p.C));
}

constexpr int kKmQueries = 128;   // queries per CTA of the distance kernel (one per thread)
constexpr int kKmCentTile = 16;   // centroids staged per step

template <int D>
struct KmeansSmem {
  static constexpr size_t Q_BYTES = static_cast<size_t>(kKmQueries) * D * 2;      // bf16, transposed
  static constexpr size_t C_BYTES = static_cast<size_t>(kKmCentTile) * D * 8;     // fp64 centroids
  static constexpr size_t BYTES = Q_BYTES + C_BYTES;
};

// Squared distances of 128 queries to every centroid: with ALL = false, the index of the nearest
// (ties to the lower centroid) into assign; with ALL = true, every distance into dist
// (centroid-major).  grid (ceil(N / 128), BH), block 128, one query per thread.
template <int D, bool ALL>
__global__ void __launch_bounds__(kKmQueries) kmeans_dist_kernel(const KmeansParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(sm);  // [D][128]: a warp reads 64 bytes
  double* cs = reinterpret_cast<double*>(sm + KmeansSmem<D>::Q_BYTES);
  const int bh = blockIdx.y, t = threadIdx.x;
  const int i0 = blockIdx.x * kKmQueries, i = i0 + t;
  const __nv_bfloat16* Qh = p.Q + static_cast<size_t>(bh) * p.N * D;
  const double* ch = p.cent + static_cast<size_t>(bh) * p.G * D;
  // the block's query rows, transposed (rows past N are zero and never written out)
  for (int e = t; e < kKmQueries * D / 8; e += kKmQueries) {
    const int r = e / (D / 8), c8 = e % (D / 8);
    const int qi = i0 + r;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (qi < p.N) v = *reinterpret_cast<const uint4*>(Qh + static_cast<size_t>(qi) * D + c8 * 8);
    const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
    for (int k = 0; k < 8; ++k) qs[(c8 * 8 + k) * kKmQueries + r] = h[k];
  }
  double best = INFINITY;
  int best_g = 0;
  for (int g0 = 0; g0 < p.G; g0 += kKmCentTile) {
    const int ng = min(kKmCentTile, p.G - g0);
    __syncthreads();
    for (int e = t; e < ng * D; e += kKmQueries) cs[e] = ch[static_cast<size_t>(g0) * D + e];
    __syncthreads();
    for (int gg = 0; gg < ng; ++gg) {
      double acc = 0.0;
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        const double diff = __dsub_rn(km_bf2d(qs[c * kKmQueries + t]), cs[gg * D + c]);
        acc = __dadd_rn(acc, __dmul_rn(diff, diff));
      }
      if (ALL) {
        if (i < p.N) p.dist[(static_cast<size_t>(bh) * p.G + g0 + gg) * p.N + i] = acc;
      } else if (acc < best) {
        best = acc;
        best_g = g0 + gg;
      }
    }
  }
  if (!ALL && i < p.N) p.assign[static_cast<size_t>(bh) * p.N + i] = best_g;
}

// Centroid update: the mean of the queries assigned to g, summed in query order; an empty
// cluster keeps its centroid.  grid (G, BH), block D threads (thread c owns coordinate c): the
// assignments are scanned D at a time and the window's members listed in order by ballots.
template <int D>
__global__ void __launch_bounds__(D) kmeans_update_kernel(const KmeansParams p) {
  constexpr int NW = D / 32;
  __shared__ int mem[D];
  __shared__ int wcount[NW];
  const int g = blockIdx.x, bh = blockIdx.y, c = threadIdx.x, w = c >> 5, l = c & 31;
  const int32_t* as = p.assign + static_cast<size_t>(bh) * p.N;
  const __nv_bfloat16* Qh = p.Q + static_cast<size_t>(bh) * p.N * D;
  double acc = 0.0;
  int count = 0;
  for (int b0 = 0; b0 < p.N; b0 += D) {
    const int i = b0 + c;
    const bool is = i < p.N && as[i] == g;
    const uint32_t bal = __ballot_sync(0xffffffffu, is);
    if (l == 0) wcount[w] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      before += k < w ? wcount[k] : 0;
      total += wcount[k];
    }
    if (is) mem[before + __popc(bal & ((1u << l) - 1u))] = i;
    __syncthreads();
    for (int m = 0; m < total; ++m) acc = __dadd_rn(acc, km_bf2d(Qh[static_cast<size_t>(mem[m]) * D + c]));
    count += total;
    __syncthreads();
  }
  if (count > 0) p.cent[(static_cast<size_t>(bh) * p.G + g) * D + c] = __ddiv_rn(acc, static_cast<double>(count));
}

// Order-preserving 64-bit key of a non-negative double.
__device__ __forceinline__ unsigned long long km_key(double x) {
  return static_cast<unsigned long long>(__double_as_longlong(x + 0.0));
}

// Equal sizes: clusters in order take their C nearest untaken queries (ties to the lower index).
// One CTA per head (grid BH, block 512): for each cluster, an exact radix select of the C-th
// smallest key among the untaken queries, then an order-preserving compaction of the chosen.
__global__ void __launch_bounds__(512) kmeans_balance_kernel(const KmeansParams p) {
  __shared__ int hist[256];
  __shared__ int scan[48];
  const int bh = blockIdx.x, t = threadIdx.x, w = t >> 5, l = t & 31;
  constexpr int NW = 16;
  unsigned char* tk = p.taken + static_cast<size_t>(bh) * p.N;
  int32_t* out = p.perm + static_cast<size_t>(bh) * p.N;
  for (int i = t; i < p.N; i += blockDim.x) tk[i] = 0;
  __syncthreads();
  for (int g = 0; g < p.G; ++g) {
    const double* dg = p.dist + (static_cast<size_t>(bh) * p.G + g) * p.N;
    unsigned long long prefix = 0, pmask = 0;
    int kk = p.C;
#pragma unroll 1
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      if (t < 256) hist[t] = 0;
      __syncthreads();
      for (int i = t; i < p.N; i += blockDim.x) {
        if (tk[i]) continue;
        const unsigned long long u = km_key(dg[i]);
        if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255ull], 1);
      }
      __syncthreads();
      if (w == 0) {
        int h[8], s = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          h[k] = hist[8 * l + k];
          s += h[k];
        }
        int incl = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, o);
          if (l >= o) incl += v;
        }
        const int excl = incl - s;
        if (excl < kk && kk <= incl) {
          int below = excl, digit = 8 * l;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (below + h[k] >= kk) {
              digit = 8 * l + k;
              break;
            }
            below += h[k];
          }
          scan[0] = digit;
          scan[1] = below;
        }
      }
      __syncthreads();
      prefix |= static_cast<unsigned long long>(scan[0]) << shift;
      pmask |= 255ull << shift;
      kk -= scan[1];
      __syncthreads();
    }
    // take every untaken key below T and the first kk equal to it, in query order
    const unsigned long long T = prefix;
    const int need_eq = kk;
    int out_base = 0, eq_seen = 0;
    for (int b0 = 0; b0 < p.N; b0 += blockDim.x) {
      const int i = b0 + t;
      const bool valid = i < p.N && !tk[i];
      const unsigned long long u = valid ? km_key(dg[i]) : ~0ull;
      const bool lt = valid && u < T, eq = valid && u == T;
      const uint32_t beq = __ballot_sync(0xffffffffu, eq);
      if (l == 0) scan[8 + w] = __popc(beq);
      __syncthreads();
      int eq_before = eq_seen, eq_total = 0;
      for (int k = 0; k < NW; ++k) {
        if (k < w) eq_before += scan[8 + k];
        eq_total += scan[8 + k];
      }
      eq_before += __popc(beq & ((1u << l) - 1u));
      const bool take = lt || (eq && eq_before < need_eq);
      const uint32_t bt = __ballot_sync(0xffffffffu, take);
      if (l == 0) scan[24 + w] = __popc(bt);
      __syncthreads();
      int tb = 0, ttot = 0;
      for (int k = 0; k < NW; ++k) {
        if (k < w) tb += scan[24 + k];
        ttot += scan[24 + k];
      }
      tb += __popc(bt & ((1u << l) - 1u));
      if (take) {
        out[g * p.C + out_base + tb] = i;
        tk[i] = 1;
      }
      out_base += ttot;
      eq_seen += eq_total;
      __syncthreads();
    }
    __syncthreads();
  }
}

}  // namespace mcs
