// GPTQ on the GPU: the damped Hessian and the error-compensating column sweep.
//
// "CMU 11-868 LLM Systems: Model Quantization" reading guide, §L20 "GPTQ":
// quantize one column block at a time; after each column, push its rounding
// error, divided by the diagonal element of G = Cholesky((2 X X^T + lambda I)^-1)^T,
// onto the rest of the block, and after the block onto every column right of
// it; the columns go in a fixed order.  "Learning-ML-DL ch. 11", §11.4: H = 2 X X^T
// is the Hessian of the output error of each weight row, damped by a fraction
// of its mean diagonal.
//
// Everything is float64 with one rounding per product, sum, difference and
// quotient (the _rn intrinsics), in this order:
//   group (block of 128 columns) parameters from the block as the sweep
//   reaches it: Delta = fp16((max - min) / (2^N - 1)), z = clamp(rint(-min / Delta));
//   column i: u = clamp(rint(w / Delta) + z), e = (w - (u - z) Delta) / G[i][i],
//   later columns j of the block: w_j - e G[i][j];
//   after the block, columns j right of it: w_j - (sum over the block's i, in
//   order, of e_i G[i][j]).
// Given the same G, the codes, steps and zero points are therefore the same
// bits whatever the launch shape.  Rows are independent: a warp sweeps a row
// block by block, and the update right of the block is a separate kernel.
#include "common.cuh"
#include "internal.h"

namespace w4a16 {
namespace {

// ---- H = 2 X^T X (+ lambda I, added by gptq_damp_kernel) -----------------------
// 64 x 64 tiles of H, 4 x 4 per thread, tokens in chunks of 16 staged in shared
// memory.  The fp16 products are exact in fp64; each entry adds them in token order.
constexpr int kHTile = 64;
constexpr int kHChunk = 16;

__global__ void __launch_bounds__(256) gptq_hessian_kernel(const __half* __restrict__ X, int T, int K,
                                                           double* __restrict__ H) {
  __shared__ double xa[kHChunk][kHTile];
  __shared__ double xb[kHChunk][kHTile];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int i0 = blockIdx.y * kHTile, j0 = blockIdx.x * kHTile;
  double acc[4][4] = {};
  for (int t0 = 0; t0 < T; t0 += kHChunk) {
    for (int e = threadIdx.x; e < kHChunk * kHTile; e += 256) {
      const int c = e % kHTile, t = e / kHTile;
      const bool in_t = t0 + t < T;
      xa[t][c] = (in_t && i0 + c < K) ? static_cast<double>(__half2float(X[static_cast<size_t>(t0 + t) * K + i0 + c])) : 0.0;
      xb[t][c] = (in_t && j0 + c < K) ? static_cast<double>(__half2float(X[static_cast<size_t>(t0 + t) * K + j0 + c])) : 0.0;
    }
    __syncthreads();
    for (int t = 0; t < kHChunk; ++t) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = __dadd_rn(acc[a][b], __dmul_rn(xa[t][ty * 4 + a], xb[t][tx * 4 + b]));
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int i = i0 + ty * 4 + a;
    if (i >= K) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = j0 + tx * 4 + b;
      if (j < K) H[static_cast<size_t>(i) * K + j] = 2.0 * acc[a][b];
    }
  }
}

// lambda = damp * (mean of the diagonal), the diagonal added in index order by one thread.
__global__ void gptq_damp_kernel(double* __restrict__ H, int K, double damp) {
  __shared__ double lam;
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < K; ++i) s = __dadd_rn(s, H[static_cast<size_t>(i) * K + i]);
    lam = __dmul_rn(damp, __ddiv_rn(s, static_cast<double>(K)));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < K; i += blockDim.x) {
    double* d = H + static_cast<size_t>(i) * K + i;
    *d = __dadd_rn(*d, lam);
  }
}

// ---- the sweep of one block of 128 columns ---------------------------------------
// A warp per row; lane l holds columns b0 + l + 32 m, m = 0..3.  The warp writes
// the row's codes (bytes), the block's errors e and the group's Delta and z.
constexpr int kGroupCols = 128;
constexpr int kSweepRows = 8;  // warps (rows) per CTA

struct SweepArgs {
  const __half* W;      // [N][K] fp16, read for the first block
  double* Wc;           // [N][K] working copy (columns right of the current block)
  const double* G;      // [K][K] upper-triangular factor
  uint8_t* codes;       // [N][K]
  double* errs;         // [N][128] the current block's e
  __half* scales;       // [N][K/128]
  __half* zeros;
  int N, K, bits, mode;
};

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_min(double v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__global__ void __launch_bounds__(32 * kSweepRows) gptq_block_kernel(const SweepArgs a, int b0) {
  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * kSweepRows + (threadIdx.x >> 5);
  if (r >= a.N) return;  // a whole warp leaves together
  const size_t row = static_cast<size_t>(r) * a.K;
  double w[4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const int j = b0 + lane + 32 * m;
    w[m] = b0 == 0 ? static_cast<double>(__half2float(a.W[row + j])) : a.Wc[row + j];
  }
  // group parameters from the block as it stands (max and min are exact)
  const double qmax = static_cast<double>((1 << a.bits) - 1);
  double d, z;
  if (a.mode == 0) {
    const double mx = warp_max(fmax(fmax(w[0], w[1]), fmax(w[2], w[3])));
    const double mn = warp_min(fmin(fmin(w[0], w[1]), fmin(w[2], w[3])));
    __half dh = __double2half(__ddiv_rn(__dsub_rn(mx, mn), qmax));
    if (__half2float(dh) == 0.0f) dh = __double2half(__ddiv_rn(1.0, qmax));
    d = static_cast<double>(__half2float(dh));
    z = fmin(fmax(rint(__ddiv_rn(-mn, d)), 0.0), qmax) + 0.0;
  } else {
    const double amax = warp_max(fmax(fmax(fabs(w[0]), fabs(w[1])), fmax(fabs(w[2]), fabs(w[3]))));
    const double half = static_cast<double>(1 << (a.bits - 1));
    __half dh = __double2half(__ddiv_rn(amax, half));
    if (__half2float(dh) == 0.0f) dh = __double2half(__ddiv_rn(1.0, half));
    d = static_cast<double>(__half2float(dh));
    z = half;
  }
  if (lane == 0) {
    const size_t g = static_cast<size_t>(r) * (a.K / kGroupCols) + b0 / kGroupCols;
    a.scales[g] = __double2half(d);
    a.zeros[g] = __double2half(z);
  }
  // the columns of the block, left to right
  for (int i = 0; i < kGroupCols; ++i) {
    const int owner = i & 31, slot = i >> 5;
    const double wi = __shfl_sync(0xffffffffu, slot == 0 ? w[0] : slot == 1 ? w[1] : slot == 2 ? w[2] : w[3], owner);
    const double u = fmin(fmax(__dadd_rn(rint(__ddiv_rn(wi, d)), z), 0.0), qmax);
    const double gii = __ldg(a.G + static_cast<size_t>(b0 + i) * a.K + b0 + i);
    const double e = __ddiv_rn(__dsub_rn(wi, __dmul_rn(__dsub_rn(u, z), d)), gii);
    if (lane == owner) {
      a.codes[row + b0 + i] = static_cast<uint8_t>(u);
      a.errs[static_cast<size_t>(r) * kGroupCols + i] = e;
    }
    const double* gi = a.G + static_cast<size_t>(b0 + i) * a.K + b0;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int c = lane + 32 * m;  // column within the block
      if (c > i) w[m] = __dsub_rn(w[m], __dmul_rn(e, __ldg(gi + c)));
    }
  }
}

// ---- the block's corrections to every column right of it ------------------------
// Wc[r][j] -= sum_i e[r][i] G[b0 + i][j], i = 0..127 added in order.  64 x 64
// tiles of (rows, columns), 4 x 4 per thread; e and G staged 16 columns of the
// block at a time.  For the first block, the columns come from W itself.
constexpr int kUTile = 64;
constexpr int kUChunk = 16;

__global__ void __launch_bounds__(256) gptq_update_kernel(const SweepArgs a, int b0) {
  __shared__ double es[kUChunk][kUTile];  // [i][row]
  __shared__ double gs[kUChunk][kUTile];  // [i][column]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int r0 = blockIdx.x * kUTile;
  const int b1 = b0 + kGroupCols;
  const int j0 = b1 + blockIdx.y * kUTile;
  double acc[4][4] = {};
  for (int i0 = 0; i0 < kGroupCols; i0 += kUChunk) {
    for (int e = threadIdx.x; e < kUChunk * kUTile; e += 256) {
      const int c = e % kUTile, i = e / kUTile;
      es[i][c] = r0 + c < a.N ? a.errs[static_cast<size_t>(r0 + c) * kGroupCols + i0 + i] : 0.0;
      gs[i][c] = j0 + c < a.K ? a.G[static_cast<size_t>(b0 + i0 + i) * a.K + j0 + c] : 0.0;
    }
    __syncthreads();
    for (int i = 0; i < kUChunk; ++i) {
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = __dadd_rn(acc[p][q], __dmul_rn(es[i][ty * 4 + p], gs[i][tx * 4 + q]));
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const int r = r0 + ty * 4 + p;
    if (r >= a.N) continue;
    const size_t row = static_cast<size_t>(r) * a.K;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = j0 + tx * 4 + q;
      if (j >= a.K) continue;
      const double w = b0 == 0 ? static_cast<double>(__half2float(a.W[row + j])) : a.Wc[row + j];
      a.Wc[row + j] = __dsub_rn(w, acc[p][q]);
    }
  }
}

// ---- codes -> layout v1 ------------------------------------------------------------
// Word (n, j) holds inputs 8j + i; nibble slot p holds i = {0, 2, 4, 6, 1, 3, 5, 7}[p].
__global__ void gptq_pack_kernel(const uint8_t* __restrict__ codes, long long words, uint32_t* __restrict__ qweight) {
  for (long long wi = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; wi < words;
       wi += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint8_t* c = codes + wi * 8;
    qweight[wi] = static_cast<uint32_t>(c[0]) | (static_cast<uint32_t>(c[2]) << 4) | (static_cast<uint32_t>(c[4]) << 8) |
                  (static_cast<uint32_t>(c[6]) << 12) | (static_cast<uint32_t>(c[1]) << 16) |
                  (static_cast<uint32_t>(c[3]) << 20) | (static_cast<uint32_t>(c[5]) << 24) |
                  (static_cast<uint32_t>(c[7]) << 28);
  }
}

// ---- the factor G = Cholesky(H^-1)^T ---------------------------------------------
// With P the reversal of the index order, P H P = L L^T (Cholesky), U = P L P is
// upper triangular with H = U U^T, and G = U^-1 = P L^-1 P is upper triangular
// with a positive diagonal and G^T G = H^-1: by the uniqueness of the Cholesky
// factorization it is the factor of [CMU] §L20 step 1.  fp64 throughout; the
// sums run over warp lanes, so G matches numpy's to rounding (about 1e-12
// relative at K = 4096), not bit for bit.

// A[i][j] = H[K-1-i][K-1-j] on and below the diagonal, 0 above.
__global__ void gptq_reverse_kernel(const double* __restrict__ H, int K, double* __restrict__ A) {
  const long long n = static_cast<long long>(K) * K;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(e / K), j = static_cast<int>(e % K);
    A[e] = j <= i ? H[static_cast<long long>(K - 1 - i) * K + (K - 1 - j)] : 0.0;
  }
}

// Blocked factorization in 64 x 64 tiles (K is a multiple of 128).  Right-looking
// Cholesky: for each block column kb, the diagonal tile is factored (and its
// triangular inverse formed) by one CTA, the panel below becomes
// L[ib][kb] = A[ib][kb] inv(L[kb][kb])^T, and the trailing lower triangle is
// updated, A[ib][jb] -= L[ib][kb] L[jb][kb]^T.  Then X = L^-1 by block rows:
// X[ib][ib] = inv(L[ib][ib]) and, for kb < ib,
// X[ib][kb] = -inv(L[ib][ib]) sum_{jb = kb}^{ib-1} L[ib][jb] X[jb][kb].
// Every tile product is a 64 x 64 x 64 fp64 product: 256 threads, 4 x 4
// outputs each, operands staged in shared memory with k outermost.
constexpr int kB = 64;
constexpr int kBP = kB + 2;  // padded row of a staged tile (doubles)

// dst[k][x] = src[x][k] (transpose) or src[k][x]; src row stride ld.
__device__ __forceinline__ void stage_tile(double (*dst)[kBP], const double* src, long long ld, bool transpose) {
  for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) {
    const int a = e / kB, b = e % kB;  // b runs fastest: coalesced reads of src row a
    const double v = src[static_cast<long long>(a) * ld + b];
    if (transpose)
      dst[b][a] = v;  // src[a][b] = P[x = a][k = b]
    else
      dst[a][b] = v;  // src[a][b] = Q[k = a][x = b]
  }
}

// acc[i][j] += sum_k Ps[k][4 tr + i] * Qs[k][4 tc + j]
__device__ __forceinline__ void tile_product(double (&acc)[4][4], const double (*Ps)[kBP], const double (*Qs)[kBP],
                                             int tr, int tc) {
#pragma unroll 4
  for (int k = 0; k < kB; ++k) {
    double p[4], q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      p[i] = Ps[k][4 * tr + i];
      q[i] = Qs[k][4 * tc + i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fma(p[i], q[j], acc[i][j]);
  }
}

// Diagonal tile kb: L[kb][kb] (lower) in place and Dinv[kb] = its inverse.
__global__ void __launch_bounds__(256) gptq_chol_diag_kernel(double* __restrict__ L, int K, int kb,
                                                             double* __restrict__ Dinv) {
  extern __shared__ double sm[];
  double(*a)[kB + 1] = reinterpret_cast<double(*)[kB + 1]>(sm);
  double(*x)[kB + 1] = reinterpret_cast<double(*)[kB + 1]>(sm + kB * (kB + 1));
  double* tile = L + static_cast<long long>(kb) * kB * K + static_cast<long long>(kb) * kB;
  for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) a[e / kB][e % kB] = tile[static_cast<long long>(e / kB) * K + e % kB];
  __syncthreads();
  // Column j: d = sqrt(a[j][j]) (kept at a[j][j]); the trailing lower triangle
  // takes a[i][c] -= a[i][j] a[c][j] / d^2 from the unscaled column, which is
  // divided by d only once every later column is done.  Two barriers per column.
  for (int j = 0; j < kB; ++j) {
    if (threadIdx.x == 0) a[j][j] = sqrt(a[j][j]);
    __syncthreads();
    const double inv_d2 = 1.0 / (a[j][j] * a[j][j]);
    for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) {
      const int i = e / kB, c = e % kB;
      if (c > j && c <= i) a[i][c] = fma(-a[i][j] * inv_d2, a[c][j], a[i][c]);
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) {
    const int i = e / kB, c = e % kB;
    if (i > c) a[i][c] /= a[c][c];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) {
    const int i = e / kB, c = e % kB;
    tile[static_cast<long long>(i) * K + c] = c <= i ? a[i][c] : 0.0;
  }
  // inverse by forward substitution, one column per thread
  if (threadIdx.x < kB) {
    const int c = threadIdx.x;
    for (int i = 0; i < c; ++i) x[i][c] = 0.0;
    x[c][c] = 1.0 / a[c][c];
    for (int i = c + 1; i < kB; ++i) {
      double sum = 0.0;
      for (int k = c; k < i; ++k) sum = fma(a[i][k], x[k][c], sum);
      x[i][c] = -sum / a[i][i];
    }
  }
  __syncthreads();
  double* dinv = Dinv + static_cast<long long>(kb) * kB * kB;
  for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) dinv[e] = x[e / kB][e % kB];
}

// Panel of block column kb: block row ib = kb + 1 + blockIdx.x,
// L[ib][kb] = A[ib][kb] Dinv[kb]^T.
__global__ void __launch_bounds__(256) gptq_chol_panel_kernel(double* __restrict__ L, int K, int kb,
                                                              const double* __restrict__ Dinv) {
  extern __shared__ double sm[];
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  const int ib = kb + 1 + blockIdx.x;
  double* tile = L + static_cast<long long>(ib) * kB * K + static_cast<long long>(kb) * kB;
  stage_tile(Ps, tile, K, true);                                           // P[r][k] = A[ib][kb][r][k]
  stage_tile(Qs, Dinv + static_cast<long long>(kb) * kB * kB, kB, true);   // Q[k][c] = Dinv[c][k]
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product(acc, Ps, Qs, tr, tc);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tile[static_cast<long long>(4 * tr + i) * K + 4 * tc + j] = acc[i][j];
}

// Trailing update after block column kb: tile (ib, jb) with kb < jb <= ib, numbered
// row by row over the lower triangle; A[ib][jb] -= L[ib][kb] L[jb][kb]^T.
__global__ void __launch_bounds__(256) gptq_chol_update_kernel(double* __restrict__ L, int K, int kb) {
  extern __shared__ double sm[];
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  // blockIdx.x = t (t + 1) / 2 + c for tile row t, column c <= t of the trailing triangle
  const int b = blockIdx.x;
  int t = static_cast<int>((sqrt(8.0 * b + 1.0) - 1.0) / 2.0);
  while ((t + 1) * (t + 2) / 2 <= b) ++t;
  while (t * (t + 1) / 2 > b) --t;
  const int c = b - t * (t + 1) / 2;
  const int ib = kb + 1 + t, jb = kb + 1 + c;
  stage_tile(Ps, L + static_cast<long long>(ib) * kB * K + static_cast<long long>(kb) * kB, K, true);
  stage_tile(Qs, L + static_cast<long long>(jb) * kB * K + static_cast<long long>(kb) * kB, K, true);
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product(acc, Ps, Qs, tr, tc);
  double* tile = L + static_cast<long long>(ib) * kB * K + static_cast<long long>(jb) * kB;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double* d = tile + static_cast<long long>(4 * tr + i) * K + 4 * tc + j;
      *d -= acc[i][j];
    }
}

// X = L^-1 by right-looking forward substitution on block rows, X in place of
// the remaining right-hand side R (L X = I): at step jb, block row jb is final,
// X[jb][kb] = Dinv[jb] R[jb][kb] for kb < jb and X[jb][jb] = Dinv[jb]; then every
// later block row is updated, R[ib][kb] -= L[ib][jb] X[jb][kb] for kb <= jb < ib
// (R starts as the identity: its first update, at jb = kb, is a plain product).
// Each step is parallel over its tiles, so the critical path is 2 K / 64 launches.
__global__ void __launch_bounds__(256) gptq_trinv_final_kernel(int K, int jb, const double* __restrict__ Dinv,
                                                               double* __restrict__ X) {
  extern __shared__ double sm[];
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  const int kb = blockIdx.x;  // 0 .. jb
  double* tile = X + static_cast<long long>(jb) * kB * K + static_cast<long long>(kb) * kB;
  const double* dinv = Dinv + static_cast<long long>(jb) * kB * kB;
  if (kb == jb) {
    for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) tile[static_cast<long long>(e / kB) * K + e % kB] = dinv[e];
    return;
  }
  stage_tile(Ps, dinv, kB, true);    // P[r][k] = Dinv[jb][r][k]
  stage_tile(Qs, tile, K, false);    // Q[k][c] = R[jb][kb][k][c]
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product(acc, Ps, Qs, tr, tc);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tile[static_cast<long long>(4 * tr + i) * K + 4 * tc + j] = acc[i][j];
}

// Update after step jb: CTA (blockIdx.x = kb <= jb, blockIdx.y = ib - jb - 1).
__global__ void __launch_bounds__(256) gptq_trinv_update_kernel(const double* __restrict__ L, int K, int jb,
                                                                double* __restrict__ X) {
  extern __shared__ double sm[];
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  const int kb = blockIdx.x, ib = jb + 1 + blockIdx.y;
  stage_tile(Ps, L + static_cast<long long>(ib) * kB * K + static_cast<long long>(jb) * kB, K, true);   // L[ib][jb]
  stage_tile(Qs, X + static_cast<long long>(jb) * kB * K + static_cast<long long>(kb) * kB, K, false);  // X[jb][kb]
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product(acc, Ps, Qs, tr, tc);
  double* tile = X + static_cast<long long>(ib) * kB * K + static_cast<long long>(kb) * kB;
  const bool first = kb == jb;  // R[ib][kb] is still the zero block of the identity
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double* d = tile + static_cast<long long>(4 * tr + i) * K + 4 * tc + j;
      *d = first ? -acc[i][j] : *d - acc[i][j];
    }
}

// G[K-1-i][K-1-j] = X[i][j] on and below the diagonal of X, 0 elsewhere.
__global__ void gptq_reverse_out_kernel(const double* __restrict__ X, int K, double* __restrict__ G) {
  const long long n = static_cast<long long>(K) * K;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int gi = static_cast<int>(e / K), gj = static_cast<int>(e % K);
    const int i = K - 1 - gi, j = K - 1 - gj;
    G[e] = j <= i ? X[static_cast<long long>(i) * K + j] : 0.0;
  }
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

size_t gptq_factor_workspace_bytes(int K) {
  return 2 * align256(static_cast<size_t>(K) * K * 8) + align256(static_cast<size_t>(K) * kB * 8);
}

cudaError_t launch_gptq_factor(const double* H, int K, double* G, void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* L = reinterpret_cast<double*>(ws);
  double* X = reinterpret_cast<double*>(ws + align256(static_cast<size_t>(K) * K * 8));
  double* Dinv = reinterpret_cast<double*>(ws + 2 * align256(static_cast<size_t>(K) * K * 8));
  const int nb = K / kB;
  const int smem = 2 * kB * kBP * 8, smem_diag = 2 * kB * (kB + 1) * 8;
  cudaError_t e = ensure_func_attr(reinterpret_cast<const void*>(gptq_chol_diag_kernel),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem_diag);
  if (e == cudaSuccess)
    e = ensure_func_attr(reinterpret_cast<const void*>(gptq_chol_panel_kernel),
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = ensure_func_attr(reinterpret_cast<const void*>(gptq_chol_update_kernel),
                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = ensure_func_attr(reinterpret_cast<const void*>(gptq_trinv_final_kernel),
                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e == cudaSuccess)
    e = ensure_func_attr(reinterpret_cast<const void*>(gptq_trinv_update_kernel),
                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  gptq_reverse_kernel<<<4 * device_sm_count(), 256, 0, st>>>(H, K, L);
  for (int kb = 0; kb < nb && e == cudaSuccess; ++kb) {
    gptq_chol_diag_kernel<<<1, 256, smem_diag, st>>>(L, K, kb, Dinv);
    const int m = nb - 1 - kb;
    if (m > 0) {
      gptq_chol_panel_kernel<<<m, 256, smem, st>>>(L, K, kb, Dinv);
      gptq_chol_update_kernel<<<m * (m + 1) / 2, 256, smem, st>>>(L, K, kb);
    }
    e = cudaGetLastError();
  }
  for (int jb = 0; jb < nb && e == cudaSuccess; ++jb) {
    gptq_trinv_final_kernel<<<jb + 1, 256, smem, st>>>(K, jb, Dinv, X);
    if (jb + 1 < nb) gptq_trinv_update_kernel<<<dim3(jb + 1, nb - 1 - jb), 256, smem, st>>>(L, K, jb, X);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  gptq_reverse_out_kernel<<<4 * device_sm_count(), 256, 0, st>>>(X, K, G);
  return cudaGetLastError();
}

cudaError_t launch_gptq_hessian(const __half* X, int T, int K, double damp, double* H, cudaStream_t st) {
  const dim3 grid((K + kHTile - 1) / kHTile, (K + kHTile - 1) / kHTile);
  gptq_hessian_kernel<<<grid, 256, 0, st>>>(X, T, K, H);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gptq_damp_kernel<<<1, 256, 0, st>>>(H, K, damp);
  return cudaGetLastError();
}

size_t gptq_sweep_workspace_bytes(int N, int K) {
  return align256(static_cast<size_t>(N) * K * 8) + align256(static_cast<size_t>(N) * K) +
         align256(static_cast<size_t>(N) * kGroupCols * 8);
}

cudaError_t launch_gptq_sweep(const __half* W, const double* G, int N, int K, int bits, int mode, uint32_t* qweight,
                              __half* scales, __half* zeros, void* workspace, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  SweepArgs a;
  a.W = W;
  a.G = G;
  a.Wc = reinterpret_cast<double*>(ws);
  a.codes = ws + align256(static_cast<size_t>(N) * K * 8);
  a.errs = reinterpret_cast<double*>(a.codes + align256(static_cast<size_t>(N) * K));
  a.scales = scales;
  a.zeros = zeros;
  a.N = N;
  a.K = K;
  a.bits = bits;
  a.mode = mode;
  const int sweep_grid = (N + kSweepRows - 1) / kSweepRows;
  for (int b0 = 0; b0 < K; b0 += kGroupCols) {
    gptq_block_kernel<<<sweep_grid, 32 * kSweepRows, 0, st>>>(a, b0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int right = K - (b0 + kGroupCols);
    if (right > 0) {
      const dim3 grid((N + kUTile - 1) / kUTile, (right + kUTile - 1) / kUTile);
      gptq_update_kernel<<<grid, 256, 0, st>>>(a, b0);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  const long long words = static_cast<long long>(N) * (K / 8);
  const long long blocks = (words + 255) / 256;
  const int pgrid = static_cast<int>(blocks < 8 * device_sm_count() ? blocks : 8 * device_sm_count());
  gptq_pack_kernel<<<pgrid, 256, 0, st>>>(a.codes, words, qweight);
  return cudaGetLastError();
}

}  // namespace w4a16
