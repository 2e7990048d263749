// Fast PDDP: tile-aligned query grouping by median-split principal-direction partitioning.
//
// "MC-Sparse가 확산 트랜스포머 희소 어텐션의 품질 격차를 좁힌다", section 어떻게 쓰나: groups have exactly
// the kernel's query-tile size C; a node is projected onto its principal direction and split
// at the median, recursively; the GPU version processes every node of one tree depth across
// all heads at once with batched power iteration and passes only query-index arrays between
// levels.
//
// Readings fixed where the page is silent (identical to the fp64 oracle): centered data; power
// iteration from v0 = 1/sqrt(d) for exactly 20 steps (v kept if X_c^T X_c v = 0); v's sign
// makes its largest-magnitude component (lowest index on a tie) positive; a node with m groups
// sends its floor(m/2)*C smallest projections (ties to the lower query index) to the left
// child.  All arithmetic is fp64, so the partition matches the oracle's exactly except where
// two projections agree to ~1e-13.
//
// The tree depends only on G, so every kernel runs on a (G, B*H) grid: slot g finds its node
// at the current depth by walking down from the root, and only node (or chunk) leaders work.
// Per depth: (1) chunk sums, (2) node mean + centered Gram (fully for nodes of <= CG groups,
// as chunk partials otherwise), (3) Gram reduction + power iteration for multi-chunk nodes,
// (4) projection, exact rank-r radix select on the fp64 keys and a stable partition into the
// next index array.  Members of every node stay in ascending query order, so position order
// is query-index order and leaves come out sorted.
#pragma once

#include "sm100.cuh"

namespace mcs {

constexpr int kPddpIters = 20;
constexpr int kChunkGroups = 8;  // CG: groups per Gram chunk for large nodes

struct PddpParams {
  const __nv_bfloat16* Q;  // [BH, N, d]
  const int32_t* cur;      // [BH, N] members of every node, node by node
  int32_t* nxt;            // [BH, N]
  double* psum;            // [BH, nslots, d]
  double* pgram;           // [BH, nslots, gram_elems]
  double* mu;              // [BH, G, d]   indexed by node start group
  double* vdir;            // [BH, G, d]
  unsigned long long* keys;  // [BH, N]
  int BH, N, C, G, d, level, nslots, gram_elems;
};

__device__ __forceinline__ void pddp_node_of(int g, int G, int level, int& lo, int& m) {
  lo = 0;
  m = G;
  for (int l = 0; l < level && m > 1; ++l) {
    const int h = m >> 1;
    if (g < lo + h) {
      m = h;
    } else {
      lo += h;
      m -= h;
    }
  }
}

// Slot of the Gram chunk of node [lo, lo+m) that lies in aligned block b (m > CG only).
__device__ __forceinline__ int pddp_slot(int b, int lo) {
  return 2 * b + ((b == lo / kChunkGroups && lo > b * kChunkGroups) ? 1 : 0);
}

__device__ __forceinline__ double bf2d(__nv_bfloat16 x) { return static_cast<double>(__bfloat162float(x)); }

// Order-preserving map of a double to uint64 (-0 is folded into +0 first).
__device__ __forceinline__ unsigned long long orderable(double x) {
  x = x + 0.0;
  unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}

// ---------------------------------------------------------------------------------------
__global__ void pddp_init_kernel(int32_t* perm, int N, long long total) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    perm[i] = static_cast<int32_t>(i % N);
}

// (1) chunk sums for nodes with more than CG groups.  blockDim = 128 (>= d).
__global__ void pddp_sum_kernel(const PddpParams p) {
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  int lo, m;
  pddp_node_of(g, p.G, p.level, lo, m);
  if (m <= kChunkGroups) return;
  const int b = g / kChunkGroups;
  const int g0 = max(lo, b * kChunkGroups);
  if (g != g0) return;
  const int g1 = min((b + 1) * kChunkGroups, lo + m);
  if (t >= p.d) return;
  const int32_t* members = p.cur + static_cast<size_t>(bh) * p.N;
  const __nv_bfloat16* Qh = p.Q + static_cast<size_t>(bh) * p.N * p.d;
  double s = 0.0;
  for (int r = g0 * p.C; r < g1 * p.C; ++r) s += bf2d(Qh[static_cast<size_t>(members[r]) * p.d + t]);
  p.psum[(static_cast<size_t>(bh) * p.nslots + pddp_slot(b, lo)) * p.d + t] = s;
}

// Gram accumulation layout: 256 threads, thread t = (ti, tj) = (t % 16, t / 16) owns entry
// (16*bi + ti, 16*bj + tj) of every upper 16x16 block bi <= bj (NB = D/16 blocks per side,
// NB*(NB+1)/2 blocks: 36 at d = 128).  Within a warp ti covers 16 consecutive columns of a
// staged row and tj two values, so every shared-memory read is conflict-free or a broadcast.
template <int D>
struct GramLayout {
  static constexpr int NB = D / 16;
  static constexpr int NUB = NB * (NB + 1) / 2;  // upper blocks
  static constexpr int RB = 32;                  // rows staged per batch
  static constexpr int UT = D * (D + 1) / 2;     // packed upper-triangle length
};

__device__ __forceinline__ int ut_index(int r, int c, int D) {  // r <= c
  return r * D - r * (r - 1) / 2 + (c - r);
}

// acc[u] += sum over rows [r0, r1) of (x - mu)[16*bi+ti] * (x - mu)[16*bj+tj], u = (bi, bj)
template <int D>
__device__ __forceinline__ void gram_rows(const __nv_bfloat16* Qh, const int32_t* members, int r0, int r1,
                                          const double* mu_s, double* xs, double (&acc)[GramLayout<D>::NUB]) {
  constexpr int NB = GramLayout<D>::NB, NUB = GramLayout<D>::NUB, RB = GramLayout<D>::RB;
  const int t = threadIdx.x, ti = t & 15, tj = t >> 4;
#pragma unroll
  for (int u = 0; u < NUB; ++u) acc[u] = 0.0;
  for (int rb = r0; rb < r1; rb += RB) {
    const int nr = min(RB, r1 - rb);
    __syncthreads();
    for (int e = t; e < nr * D; e += 256) {
      const int r = e / D, c = e - r * D;
      xs[r * D + c] = bf2d(Qh[static_cast<size_t>(members[rb + r]) * D + c]) - mu_s[c];
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      double av[NB], bv[NB];
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        av[i] = xs[r * D + 16 * i + ti];
        bv[i] = xs[r * D + 16 * i + tj];
      }
      int u = 0;
#pragma unroll
      for (int bi = 0; bi < NB; ++bi)
#pragma unroll
        for (int bj = bi; bj < NB; ++bj) {
          acc[u] = fma(av[bi], bv[bj], acc[u]);
          ++u;
        }
    }
  }
}

// Power iteration on the full symmetric Gram matrix G_s [D][D] (fp64, shared), 256 threads.
// Writes the sign-fixed unit vector to v_s[D].
template <int D>
__device__ __forceinline__ void power_iterate(const double* G_s, double* v_s, double* w_s, double* red) {
  const int t = threadIdx.x;
  const double v0 = 1.0 / sqrt(static_cast<double>(D));
  if (t < D) v_s[t] = v0;
  __syncthreads();
  for (int it = 0; it < kPddpIters; ++it) {
    double w = 0.0;
    if (t < D) {
      for (int b = 0; b < D; ++b) w = fma(G_s[b * D + t], v_s[b], w);
      w_s[t] = w;
    }
    // deterministic norm^2: fixed shuffle tree per warp, then warps in order
    double sq = t < D ? w * w : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_down_sync(0xffffffffu, sq, o);
    if ((t & 31) == 0) red[t >> 5] = sq;
    __syncthreads();
    if (t == 0) {
      double s = 0.0;
      for (int i = 0; i < (D + 31) / 32; ++i) s += red[i];
      red[16] = s;
    }
    __syncthreads();
    const double n2 = red[16];
    if (n2 == 0.0) break;  // X_c^T X_c v = 0: keep v
    const double nrm = sqrt(n2);
    if (t < D) v_s[t] = w_s[t] / nrm;
    __syncthreads();
  }
  __syncthreads();
  if (t == 0) {
    int jm = 0;
    double am = fabs(v_s[0]);
    for (int j = 1; j < D; ++j) {
      const double a = fabs(v_s[j]);
      if (a > am) {
        am = a;
        jm = j;
      }
    }
    red[17] = v_s[jm] < 0.0 ? -1.0 : 1.0;
  }
  __syncthreads();
  if (t < D) v_s[t] *= red[17];
  __syncthreads();
}

// The chunks of node [lo, lo+m) at the current depth: nodes of <= CG groups are one chunk
// (leader lo); larger nodes are cut at multiples of CG groups (leaders max(lo, b*CG)).  Each
// chunk's partial Gram lives in the slot of its leader group.
__device__ __forceinline__ bool pddp_chunk_of(int g, int lo, int m, int& g0, int& g1) {
  if (m <= kChunkGroups) {
    g0 = lo;
    g1 = lo + m;
  } else {
    const int b = g / kChunkGroups;
    g0 = max(lo, b * kChunkGroups);
    g1 = min((b + 1) * kChunkGroups, lo + m);
  }
  return g == g0;
}

template <int D>
struct PddpGramSmem {
  static constexpr size_t BYTES = GramLayout<D>::RB * D * 8 + D * 8;  // staging + mean
};

// (2) centered Gram partial of one chunk (upper triangle, packed) into the slot of its leader
// group; the node mean comes from the chunk sums (nodes of > CG groups) or from a direct pass
// (smaller nodes, which also store it for the split).  blockDim = 256.
template <int D>
__global__ void __launch_bounds__(256, 2) pddp_gram_kernel(const PddpParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int NB = GramLayout<D>::NB, NUB = GramLayout<D>::NUB;
  double* xs = reinterpret_cast<double*>(sm);
  double* mu_s = xs + GramLayout<D>::RB * D;
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int ti = t & 15, tj = t >> 4;
  int lo, m;
  pddp_node_of(g, p.G, p.level, lo, m);
  if (m == 1) return;
  int g0, g1;
  if (!pddp_chunk_of(g, lo, m, g0, g1)) return;
  const int32_t* members = p.cur + static_cast<size_t>(bh) * p.N;
  const __nv_bfloat16* Qh = p.Q + static_cast<size_t>(bh) * p.N * D;
  const double inv_n = 1.0 / static_cast<double>(m * p.C);
  if (t < D) {
    double s = 0.0;
    if (m <= kChunkGroups) {
      for (int r = lo * p.C; r < (lo + m) * p.C; ++r) s += bf2d(Qh[static_cast<size_t>(members[r]) * D + t]);
    } else {
      for (int bb = lo / kChunkGroups; bb <= (lo + m - 1) / kChunkGroups; ++bb)
        s += p.psum[(static_cast<size_t>(bh) * p.nslots + pddp_slot(bb, lo)) * D + t];
    }
    mu_s[t] = s * inv_n;
    if (g == lo) p.mu[(static_cast<size_t>(bh) * p.G + lo) * D + t] = s * inv_n;
  }
  __syncthreads();
  double acc[NUB];
  gram_rows<D>(Qh, members, g0 * p.C, g1 * p.C, mu_s, xs, acc);
  double* dst = p.pgram + (static_cast<size_t>(bh) * p.G + g) * p.gram_elems;
  int u = 0;
#pragma unroll
  for (int bi = 0; bi < NB; ++bi)
#pragma unroll
    for (int bj = bi; bj < NB; ++bj) {
      const int r = 16 * bi + ti, c = 16 * bj + tj;
      if (r <= c) dst[ut_index(r, c, D)] = acc[u];  // (the lower half of diagonal blocks repeats)
      ++u;
    }
}

template <int D>
struct PddpPowerSmem {
  static constexpr size_t BYTES = static_cast<size_t>(D) * D * 8 + 3 * D * 8 + 32 * 8;
};

// (3) per node: sum its chunks' partial Grams (chunk order), power iteration, store v.
template <int D>
__global__ void __launch_bounds__(256) pddp_power_kernel(const PddpParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  double* G_s = reinterpret_cast<double*>(sm);
  double* v_s = G_s + D * D;
  double* w_s = v_s + D;
  double* red = w_s + D;
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  int lo, m;
  pddp_node_of(g, p.G, p.level, lo, m);
  if (m == 1 || g != lo) return;
  const double* base = p.pgram + static_cast<size_t>(bh) * p.G * p.gram_elems;
  for (int e = t; e < D * D; e += blockDim.x) {
    const int r = e / D, c = e - r * D;
    const int u = r <= c ? ut_index(r, c, D) : ut_index(c, r, D);
    double acc = 0.0;
    if (m <= kChunkGroups) {
      acc = base[static_cast<size_t>(lo) * p.gram_elems + u];
    } else {
      for (int bb = lo / kChunkGroups; bb <= (lo + m - 1) / kChunkGroups; ++bb) {
        const int gl = max(lo, bb * kChunkGroups);
        acc += base[static_cast<size_t>(gl) * p.gram_elems + u];
      }
    }
    G_s[e] = acc;
  }
  __syncthreads();
  power_iterate<D>(G_s, v_s, w_s, red);
  if (t < D) p.vdir[(static_cast<size_t>(bh) * p.G + lo) * D + t] = v_s[t];
}

// (4) projection, exact rank split and stable partition.  blockDim = 512 (16 warps).
template <int D>
__global__ void __launch_bounds__(512) pddp_split_kernel(const PddpParams p) {
  __shared__ double mu_s[D], v_s[D];
  __shared__ int hist[256];
  __shared__ int scan[40];
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int w = t >> 5, l = t & 31;
  int lo, m;
  pddp_node_of(g, p.G, p.level, lo, m);
  if (g != lo) return;
  const size_t hoff = static_cast<size_t>(bh) * p.N;
  const int s0 = lo * p.C, n = m * p.C;
  const int32_t* cur = p.cur + hoff + s0;
  int32_t* nxt = p.nxt + hoff + s0;
  if (m == 1) {
    for (int i = t; i < n; i += blockDim.x) nxt[i] = cur[i];
    return;
  }
  if (t < D) {
    const size_t o = (static_cast<size_t>(bh) * p.G + lo) * D + t;
    mu_s[t] = p.mu[o];
    v_s[t] = p.vdir[o];
  }
  __syncthreads();
  const __nv_bfloat16* Qh = p.Q + hoff * D;
  unsigned long long* keys = p.keys + hoff + s0;
  for (int i = t; i < n; i += blockDim.x) {
    const uint4* row = reinterpret_cast<const uint4*>(Qh + static_cast<size_t>(cur[i]) * D);
    double acc = 0.0;
#pragma unroll 4
    for (int c8 = 0; c8 < D / 8; ++c8) {
      const uint4 u = row[c8];
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(h2[e]);
        acc = fma(static_cast<double>(f.x) - mu_s[8 * c8 + 2 * e], v_s[8 * c8 + 2 * e], acc);
        acc = fma(static_cast<double>(f.y) - mu_s[8 * c8 + 2 * e + 1], v_s[8 * c8 + 2 * e + 1], acc);
      }
    }
    keys[i] = orderable(acc);
  }
  __syncthreads();
  // radix select: the r-th smallest key (1-based), 8 passes of 8 bits
  const int r = (m >> 1) * p.C;
  unsigned long long prefix = 0, pmask = 0;
  int kk = r;
#pragma unroll 1
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    if (t < 256) hist[t] = 0;
    __syncthreads();
    for (int i = t; i < n; i += blockDim.x) {
      const unsigned long long u = keys[i];
      if ((u & pmask) == prefix) atomicAdd(&hist[(u >> shift) & 255ull], 1);
    }
    __syncthreads();
    if (w == 0) {
      int h[8], s = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        h[i] = hist[8 * l + i];
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
        int below = excl, digit = 8 * l;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (below + h[i] >= kk) {
            digit = 8 * l + i;
            break;
          }
          below += h[i];
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
  const unsigned long long T = prefix;
  const int need_eq = kk;
  int left_base = 0, right_base = 0, eq_seen = 0;
  constexpr int NW = 16;
  for (int base = 0; base < n; base += blockDim.x) {
    const int i = base + t;
    const bool valid = i < n;
    const unsigned long long u = valid ? keys[i] : ~0ull;
    const bool lt = valid && u < T;
    const bool eq = valid && u == T;
    const uint32_t beq = __ballot_sync(0xffffffffu, eq);
    if (l == 0) scan[8 + w] = __popc(beq);
    __syncthreads();
    int eq_before = eq_seen, eq_total = 0;
    for (int i2 = 0; i2 < NW; ++i2) {
      if (i2 < w) eq_before += scan[8 + i2];
      eq_total += scan[8 + i2];
    }
    eq_before += __popc(beq & ((1u << l) - 1u));
    const bool left = lt || (eq && eq_before < need_eq);
    const uint32_t bl = __ballot_sync(0xffffffffu, left);
    if (l == 0) scan[24 + w] = __popc(bl);
    __syncthreads();
    int lb = 0, ltot = 0;
    for (int i2 = 0; i2 < NW; ++i2) {
      if (i2 < w) lb += scan[24 + i2];
      ltot += scan[24 + i2];
    }
    lb += __popc(bl & ((1u << l) - 1u));
    if (valid) {
      const int q = cur[i];
      if (left) nxt[left_base + lb] = q;
      else nxt[r + right_base + (t - lb)] = q;
    }
    const int nvalid = min(static_cast<int>(blockDim.x), n - base);
    left_base += ltot;
    right_base += nvalid - ltot;
    eq_seen += eq_total;
    __syncthreads();
  }
}

}  // namespace mcs
