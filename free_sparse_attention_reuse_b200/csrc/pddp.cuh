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
// Per depth: (1) uncentered Gram X^T X and column sums of every chunk (a whole node of <= CG
// groups, else CG-group pieces) of the root and of every left child, the Gram on the fp64
// tensor cores at d = 128; (2) per node: its uncentered Gram and sums, the chunk reduction for
// a left child or the root, and for a right child its parent's (kept from the level above)
// less its left sibling's, since the two children partition the parent's rows (when that
// sibling splits too, so that its chunks are there), which leaves 56 % of the Gram rows of a
// 252-group tree to read; centring X_c^T X_c = X^T X - s s^T / n,
// mean, power iteration; (3)
// projection, exact rank-r radix select on the fp64 keys and a stable partition into the next
// index array.  Members of every node stay in ascending query order, so position order
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
  double* psum;            // [BH, G, d]   column sums of each chunk, by chunk-leader group
  double* pgram;           // [BH, G, gram_elems] uncentered Gram of each chunk, by chunk-leader group
  double* nsum;            // [BH, G, d]   column sums of a node, in slot lo + m/2 (its right child's start)
  double* ngram;           // [BH, G, gram_elems] uncentered Gram of a node, same slot
  double* mu;              // [BH, G, d]   indexed by node start group
  double* vdir;            // [BH, G, d]
  unsigned long long* keys;  // [BH, N]
  int BH, N, C, G, d, level, gram_elems;
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

// The same walk, also telling whether the node is the right child of its parent (plo, pm);
// false at the root.
__device__ __forceinline__ void pddp_node_side(int g, int G, int level, int& lo, int& m, bool& right, int& plo,
                                               int& pm) {
  lo = 0;
  m = G;
  right = false;
  plo = 0;
  pm = G;
  for (int l = 0; l < level && m > 1; ++l) {
    const int h = m >> 1;
    plo = lo;
    pm = m;
    if (g < lo + h) {
      m = h;
      right = false;
    } else {
      lo += h;
      m -= h;
      right = true;
    }
  }
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

// acc[u] += sum over rows [r0, r1) of x[16*bi+ti] * x[16*bj+tj], u = (bi, bj) (uncentered);
// csum += the staged values of this thread's column (threadIdx.x % D)
template <int D>
__device__ __forceinline__ void gram_rows(const __nv_bfloat16* Qh, const int32_t* members, int r0, int r1,
                                          double* xs, double (&acc)[GramLayout<D>::NUB], double& csum) {
  constexpr int NB = GramLayout<D>::NB, NUB = GramLayout<D>::NUB, RB = GramLayout<D>::RB;
  const int t = threadIdx.x, ti = t & 15, tj = t >> 4;
#pragma unroll
  for (int u = 0; u < NUB; ++u) acc[u] = 0.0;
  for (int rb = r0; rb < r1; rb += RB) {
    const int nr = min(RB, r1 - rb);
    __syncthreads();
    for (int e = t; e < nr * D; e += 256) {
      const int r = e / D, c = e - r * D;
      const double x = bf2d(Qh[static_cast<size_t>(members[rb + r]) * D + c]);
      xs[r * D + c] = x;
      csum += x;
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

// ---------------------------------------------------------------- fp64 tensor-core Gram (d = 128)
// D[8x8] += A[8x4] B[4x8] in fp64 on the tensor cores (mma.sync m8n8k4; there is no tcgen05
// form for fp64).  Fragments: a = A[lane/4][lane%4], b = B[lane%4][lane/4],
// c/d = C[lane/4][2*(lane%4) + {0,1}].
__device__ __forceinline__ void dmma_8x8x4(double& d0, double& d1, double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

constexpr int kGramTcStride = 128 + 8;  // staged row stride (doubles): 4 rows hit distinct banks
constexpr int kGramTcRows = 32;         // rows staged per batch

// Upper-triangle 8x8 tiles (I <= J) of the centered Gram of rows [r0, r1) (d = 128), by the
// 8 warps: warp w owns tile rows w and 15-w, 17 tiles in all.  Tile jj of the warp's list is
// (w, w+jj) for jj < 16-w and (15-w, jj-1) after (a compile-time index into acc); each 4-row
// k-step loads the two A fragments once and one B fragment per tile.
__device__ __forceinline__ void gram_tile_of(int w, int jj, int& I, int& J) {
  const bool first = jj < 16 - w;
  I = first ? w : 15 - w;
  J = first ? w + jj : jj - 1;
}

__device__ __forceinline__ void gram_rows_tc(const __nv_bfloat16* Qh, const int32_t* members, int r0, int r1,
                                             double* xs, double (&acc)[17][2], double (&csum)[8]) {
  constexpr int D = 128, S = kGramTcStride;
  const int t = threadIdx.x, w = t >> 5, l = t & 31;
  const int rr = l & 3, cc = l >> 2;  // fragment row (data row within the k-step), column
  // staging: thread t copies 8 columns (8*(t%16) .. +7) of rows t/16 and t/16 + 16 of a batch,
  // the next batch's loads in flight while this batch's MMAs run
  const int sr = t >> 4, sc = (t & 15) * 8;
#pragma unroll
  for (int i = 0; i < 17; ++i) acc[i][0] = acc[i][1] = 0.0;
#pragma unroll
  for (int j = 0; j < 8; ++j) csum[j] = 0.0;
  auto fetch = [&](int rb, uint4 (&v)[2]) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = rb + sr + 16 * h;
      v[h] = r < r1 ? *reinterpret_cast<const uint4*>(Qh + static_cast<size_t>(members[r]) * D + sc)
                    : make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 nextv[2];
  fetch(r0, nextv);
  for (int rb = r0; rb < r1; rb += kGramTcRows) {
    const int nr = min(kGramTcRows, r1 - rb);
    __syncthreads();  // the previous batch's MMAs are done with xs
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&nextv[h]);
      double* dst = xs + (sr + 16 * h) * S + sc;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(b2[e]);
        dst[2 * e] = f.x;
        dst[2 * e + 1] = f.y;
        csum[2 * e] += f.x;
        csum[2 * e + 1] += f.y;
      }
    }
    __syncthreads();
    if (rb + kGramTcRows < r1) fetch(rb + kGramTcRows, nextv);
#pragma unroll 1
    for (int k0 = 0; k0 < nr; k0 += 4) {
      const double* row = xs + (k0 + rr) * S + cc;  // rows past nr are zero
      const double a0 = row[w * 8], a1 = row[(15 - w) * 8];
#pragma unroll
      for (int jj = 0; jj < 17; ++jj) {
        int I, J;
        gram_tile_of(w, jj, I, J);
        dmma_8x8x4(acc[jj][0], acc[jj][1], I == w ? a0 : a1, row[J * 8]);
      }
    }
  }
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

// A right child whose left sibling splits too (so that the sibling's chunk partials exist at
// this depth) takes its totals from its parent's, "derived"; every other node sums its chunks.
__device__ __forceinline__ bool pddp_derived(bool right, int pm) { return right && (pm >> 1) >= 2; }

template <int D>
struct PddpGramSmem {
  // staging (padded rows on the tensor-core path at d = 128) + 256 partial column sums
  static constexpr size_t BYTES =
      (D == 128 ? static_cast<size_t>(kGramTcRows) * kGramTcStride : static_cast<size_t>(GramLayout<D>::RB) * D) * 8 +
      256 * 8;
};

// (1) uncentered Gram X^T X (upper triangle, packed) and column sums of one chunk into the
// slots of its leader group; the power kernel reduces a node's chunks and centres.
// blockDim = 256.
template <int D>
__global__ void __launch_bounds__(256, 2) pddp_gram_kernel(const PddpParams p) {
  extern __shared__ __align__(16) uint8_t sm[];
  constexpr int NB = GramLayout<D>::NB, NUB = GramLayout<D>::NUB;
  double* xs = reinterpret_cast<double*>(sm);
  double* part = xs + (D == 128 ? kGramTcRows * kGramTcStride : GramLayout<D>::RB * D);  // 256 partial sums
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  const int ti = t & 15, tj = t >> 4;
  int lo, m, plo, pm;
  bool right;
  pddp_node_side(g, p.G, p.level, lo, m, right, plo, pm);
  if (m == 1 || pddp_derived(right, pm)) return;  // its Gram is its parent's less its sibling's
  int g0, g1;
  if (!pddp_chunk_of(g, lo, m, g0, g1)) return;
  const int32_t* members = p.cur + static_cast<size_t>(bh) * p.N;
  const __nv_bfloat16* Qh = p.Q + static_cast<size_t>(bh) * p.N * D;
  double* dst = p.pgram + (static_cast<size_t>(bh) * p.G + g) * p.gram_elems;
  double csum = 0.0;
  // the chunk's column sums, in a fixed order: thread t staged column t % D
  auto store_sums = [&]() {
    part[t] = csum;
    __syncthreads();
    if (t < D) {
      double s = 0.0;
      for (int i = t; i < 256; i += D) s += part[i];
      p.psum[(static_cast<size_t>(bh) * p.G + g) * D + t] = s;
    }
  };
  if constexpr (D == 128) {
    double acc[17][2];
    double cs8[8];
    gram_rows_tc(Qh, members, g0 * p.C, g1 * p.C, xs, acc, cs8);
    // column sums: thread t staged columns 8*(t%16) .. +7; reduce the 16 threads of each
    // column group in a fixed order
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 8; ++j) xs[t * 8 + j] = cs8[j];
    __syncthreads();
    if (t < D) {
      const int c8 = t >> 3, j = t & 7;
      double s = 0.0;
      for (int q = 0; q < 16; ++q) s += xs[(q * 16 + c8) * 8 + j];
      p.psum[(static_cast<size_t>(bh) * p.G + g) * D + t] = s;
    }
    const int w = t >> 5, l = t & 31;
#pragma unroll
    for (int jj = 0; jj < 17; ++jj) {
      int I, J;
      gram_tile_of(w, jj, I, J);
      const int r = I * 8 + (l >> 2);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int c = J * 8 + (l & 3) * 2 + e;
        if (r <= c) dst[ut_index(r, c, D)] = acc[jj][e];  // (diagonal tiles hold both halves)
      }
    }
    return;
  }
  double acc[NUB];
  gram_rows<D>(Qh, members, g0 * p.C, g1 * p.C, xs, acc, csum);
  int u = 0;
#pragma unroll
  for (int bi = 0; bi < NB; ++bi)
#pragma unroll
    for (int bj = bi; bj < NB; ++bj) {
      const int r = 16 * bi + ti, c = 16 * bj + tj;
      if (r <= c) dst[ut_index(r, c, D)] = acc[u];  // (the lower half of diagonal blocks repeats)
      ++u;
    }
  store_sums();
}

// (2) per node, one CTA of 256 threads: its uncentered Gram and column sums, centred, and the
// power iteration.
//   * Totals: a derived right child starts from its parent's total (kept in slot lo) and takes
//     off its left sibling's chunks one by one; every other node adds up its own chunks in
//     chunk order.  The terms stream into shared memory with 16-byte cp.async, two in flight,
//     and every thread combines only the pieces it copied itself (no barrier in the stream).
//     A node of >= 4 groups keeps its total in slot lo + m/2 for its right child at the next
//     depth: that slot lies strictly inside the node, so it is no node's start at this depth,
//     nothing reads it here and the write races with nothing.
//   * Centring: X_c^T X_c = X^T X - s mu^T with s the column sums and mu = s / n, each entry
//     formed once from the packed triangle (min(r, c), max(r, c)), so the matrix stays exactly
//     symmetric.
//   * Power iteration from v0 = 1/sqrt(d), 20 steps, with the matrix in registers: thread
//     (rb, cb) = (2 * warp + lane / 16, lane % 16) holds rows rb + 16 i and columns cb + 16 k
//     (i, k < D/16), so the v reads of a half-warp are 16 consecutive words.  Each product
//     is finished by a butterfly over the 16 lanes of a half-warp that halves the open rows at
//     every step; the squared norm is a fixed shuffle tree per warp, then the warps in order.
//     Two barriers per step; the step stops with v kept when X_c^T X_c v = 0.
template <int D>
struct PddpPowerSmem {
  static constexpr int UT = D * (D + 1) / 2;  // packed upper triangle
  static constexpr int PIECES = UT / 2;       // 16-byte pieces of one triangle
  static constexpr int SPIECES = D / 2;       // ... of one column-sum vector
  static constexpr size_t TRI = static_cast<size_t>(UT) * 8;
  // total A, two staging triangles; total sums, two staging sum vectors; v, mu; warp partials
  static constexpr size_t BYTES = 3 * TRI + 3 * D * 8 + 2 * D * 8 + 16 * 8;
  static_assert(UT % 2 == 0 && TRI % 16 == 0, "16-byte pieces");
};

// One butterfly step over the lanes `M` apart: with C > 1 rows open, a lane keeps half of them
// (the upper half when its bit M is set) and adds its partner's half of the same rows; with one
// row left the two partners add each other's sums (the same value in both).
template <int C, int M>
__device__ __forceinline__ void pddp_butterfly(double* a, int cb) {
  if constexpr (C > 1) {
    const bool up = (cb & M) != 0;
#pragma unroll
    for (int i = 0; i < C / 2; ++i) {
      const double send = up ? a[i] : a[i + C / 2];
      const double keep = up ? a[i + C / 2] : a[i];
      a[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
    }
    pddp_butterfly<C / 2, M / 2>(a, cb);
  } else if constexpr (M >= 1) {
    a[0] = a[0] + __shfl_xor_sync(0xffffffffu, a[0], M);
    pddp_butterfly<1, M / 2>(a, cb);
  }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

template <int D>
__global__ void __launch_bounds__(256, 1) pddp_power_kernel(const PddpParams p) {
  using L = PddpPowerSmem<D>;
  constexpr int UT = L::UT, R = D / 16;
  constexpr int LR = R == 8 ? 3 : 2;  // log2 R
  static_assert(R == 4 || R == 8, "d = 64 or 128");
  extern __shared__ __align__(16) uint8_t sm[];
  double* A = reinterpret_cast<double*>(sm);
  double* B = A + UT;                  // [2][UT]
  double* sA = B + 2 * UT;             // [D]
  double* sB = sA + D;                 // [2][D]
  double* v_s = sB + 2 * D;
  double* mu_s = v_s + D;
  double* red = mu_s + D;              // [16]
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  int lo, m, plo, pm;
  bool right;
  pddp_node_side(g, p.G, p.level, lo, m, right, plo, pm);
  if (m == 1 || g != lo) return;
  const bool derived = pddp_derived(right, pm);
  const double n = static_cast<double>(m) * p.C;
  const size_t gstride = static_cast<size_t>(p.gram_elems);
  const double* cg = p.pgram + static_cast<size_t>(bh) * p.G * gstride;  // chunk partials
  const double* cs = p.psum + static_cast<size_t>(bh) * p.G * D;
  double* kg = p.ngram + static_cast<size_t>(bh) * p.G * gstride;        // kept node totals
  double* ks = p.nsum + static_cast<size_t>(bh) * p.G * D;

  // term 0: the kept parent total (derived) or the first chunk; then chunks, subtracted
  // (derived) or added
  const int clo = derived ? plo : lo, cm = derived ? (pm >> 1) : m;
  const int nchunks = cm <= kChunkGroups ? 1 : (clo + cm - 1) / kChunkGroups - clo / kChunkGroups + 1;
  const int nterms = nchunks + (derived ? 1 : 0);
  auto term_src = [&](int k, const double*& gsrc, const double*& ssrc) {
    if (derived && k == 0) {
      gsrc = kg + static_cast<size_t>(lo) * gstride;
      ssrc = ks + static_cast<size_t>(lo) * D;
      return;
    }
    const int c = k - (derived ? 1 : 0);
    const int slot = cm <= kChunkGroups ? clo : max(clo, (clo / kChunkGroups + c) * kChunkGroups);
    gsrc = cg + static_cast<size_t>(slot) * gstride;
    ssrc = cs + static_cast<size_t>(slot) * D;
  };
  auto issue = [&](int k, double* gdst, double* sdst) {
    const double *gsrc, *ssrc;
    term_src(k, gsrc, ssrc);
    const uint32_t gd = smem_u32(gdst), sd = smem_u32(sdst);
    for (int e = t; e < L::PIECES; e += 256) cp_async16(gd + e * 16, gsrc + 2 * e, 16);
    if (t < L::SPIECES) cp_async16(sd + t * 16, ssrc + 2 * t, 16);
    cp_async_commit();
  };
  issue(0, A, sA);
  if (nterms > 1) issue(1, B, sB);
  if (nterms > 2) issue(2, B + UT, sB + D);
  for (int k = 1; k < nterms; ++k) {
    if (k + 1 < nterms)
      cp_async_wait_group<1>();
    else
      cp_async_wait_group<0>();
    const int b = (k - 1) & 1;
    const double* Bb = B + b * UT;
    const double* sBb = sB + b * D;
    for (int e = t; e < L::PIECES; e += 256) {
      const double2 x = reinterpret_cast<const double2*>(Bb)[e];
      double2& a = reinterpret_cast<double2*>(A)[e];
      a = derived ? make_double2(a.x - x.x, a.y - x.y) : make_double2(a.x + x.x, a.y + x.y);
    }
    if (t < L::SPIECES) {
      const double2 x = reinterpret_cast<const double2*>(sBb)[t];
      double2& a = reinterpret_cast<double2*>(sA)[t];
      a = derived ? make_double2(a.x - x.x, a.y - x.y) : make_double2(a.x + x.x, a.y + x.y);
    }
    if (k + 2 < nterms) issue(k + 2, B + b * UT, sB + b * D);
  }
  if (nterms == 1) cp_async_wait_group<0>();
  if (m >= 4) {  // the node's total, for its right child at the next depth
    double2* kgd = reinterpret_cast<double2*>(kg + static_cast<size_t>(lo + (m >> 1)) * gstride);
    double2* ksd = reinterpret_cast<double2*>(ks + static_cast<size_t>(lo + (m >> 1)) * D);
    for (int e = t; e < L::PIECES; e += 256) kgd[e] = reinterpret_cast<const double2*>(A)[e];
    if (t < L::SPIECES) ksd[t] = reinterpret_cast<const double2*>(sA)[t];
  }
  __syncthreads();
  if (t < D) {
    const double mu = sA[t] / n;
    mu_s[t] = mu;
    p.mu[(static_cast<size_t>(bh) * p.G + lo) * D + t] = mu;
  }
  __syncthreads();

  // the thread's rows rb + 16 i and columns cb + 16 k of X_c^T X_c, into registers
  const int w = t >> 5, l = t & 31;
  const int rb = 2 * w + (l >> 4), cb = l & 15;
  double gm[R][R];
#pragma unroll
  for (int i = 0; i < R; ++i)
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int r = rb + 16 * i, c = cb + 16 * k;
      const int a = min(r, c), z = max(r, c);
      gm[i][k] = fma(-sA[a], mu_s[z], A[ut_index(a, z, D)]);
    }
  const int my_row = rb + 16 * (cb >> (4 - LR));
  const bool owner = (cb & ((1 << (4 - LR)) - 1)) == 0;
  if (t < D) v_s[t] = 1.0 / sqrt(static_cast<double>(D));
  __syncthreads();
  for (int it = 0; it < kPddpIters; ++it) {
    double vv[R], a[R];
#pragma unroll
    for (int k = 0; k < R; ++k) vv[k] = v_s[cb + 16 * k];
#pragma unroll
    for (int i = 0; i < R; ++i) {
      a[i] = 0.0;
#pragma unroll
      for (int k = 0; k < R; ++k) a[i] = fma(gm[i][k], vv[k], a[i]);
    }
    pddp_butterfly<R, 8>(a, cb);
    const double wr = a[0];
    double sq = owner ? wr * wr : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (l == 0) red[w] = sq;
    __syncthreads();  // partials complete; every read of v for this step is done
    double n2 = 0.0;
#pragma unroll
    for (int q = 0; q < 8; ++q) n2 += red[q];
    if (n2 == 0.0) break;  // X_c^T X_c v = 0: keep v (uniform: every thread read the same sum)
    if (owner) v_s[my_row] = wr / sqrt(n2);
    __syncthreads();  // v complete; every read of the partials is done
  }
  __syncthreads();
  // sign: the largest-magnitude component (lowest index on a tie) positive
  if (t == 0) {
    int jm = 0;
    double am = fabs(v_s[0]);
    for (int j = 1; j < D; ++j) {
      const double x = fabs(v_s[j]);
      if (x > am) {
        am = x;
        jm = j;
      }
    }
    red[8] = v_s[jm] < 0.0 ? -1.0 : 1.0;
  }
  __syncthreads();
  if (t < D) p.vdir[(static_cast<size_t>(bh) * p.G + lo) * D + t] = v_s[t] * red[8];
}

// (3a) projections of every row of every multi-group node onto its direction, as order-
// preserving 64-bit keys: CTA g projects the C rows at positions g*C .. g*C+C-1 (all CTAs of a
// node take part, so a large node uses many SMs).  blockDim = C.
template <int D>
__global__ void pddp_project_kernel(const PddpParams p) {
  __shared__ double mu_s[D], v_s[D];
  const int g = blockIdx.x, bh = blockIdx.y, t = threadIdx.x;
  int lo, m;
  pddp_node_of(g, p.G, p.level, lo, m);
  if (m == 1) return;
  if (t < D) {
    const size_t o = (static_cast<size_t>(bh) * p.G + lo) * D + t;
    mu_s[t] = p.mu[o];
    v_s[t] = p.vdir[o];
  }
  __syncthreads();
  const size_t hoff = static_cast<size_t>(bh) * p.N;
  const int i = g * p.C + t;  // position within the head's index array
  if (t >= p.C) return;
  const uint4* row = reinterpret_cast<const uint4*>(p.Q + (hoff + static_cast<size_t>(p.cur[hoff + i])) * D);
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
  p.keys[hoff + i] = orderable(acc);
}

// (3b) exact rank split and stable partition of each node from its keys.  blockDim = 512.
template <int D>
__global__ void __launch_bounds__(512) pddp_split_kernel(const PddpParams p) {
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
  const unsigned long long* keys = p.keys + hoff + s0;
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
