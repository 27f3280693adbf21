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
// Wc[r][j] -= sum_i e[r][i] G[b0 + i][j], i = 0..127 added in order (each
// product and each sum rounded once: the order the oracle fixes).  64 x 64 tiles
// of (rows, columns); thread (ty, tx) holds rows 4 ty + p and columns tx + 16 q,
// so that a warp's reads of G are 16 consecutive words (no bank conflicts) and
// its reads of e two broadcasts.  e and G are staged kUChunk columns of the block
// at a time, with coalesced global reads (e is row-major by row: consecutive
// threads take consecutive i of a row; the padded row keeps those stores on
// distinct banks).  For the first block, the columns come from W itself.
constexpr int kUTile = 64;
constexpr int kUChunk = 32;

__global__ void __launch_bounds__(256) gptq_update_kernel(const SweepArgs a, int b0) {
  __shared__ double es[kUChunk][kUTile + 1];  // [i][row]
  __shared__ double gs[kUChunk][kUTile];      // [i][column]
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int r0 = blockIdx.x * kUTile;
  const int b1 = b0 + kGroupCols;
  const int j0 = b1 + blockIdx.y * kUTile;
  double acc[4][4] = {};
  for (int i0 = 0; i0 < kGroupCols; i0 += kUChunk) {
    for (int e = threadIdx.x; e < kUChunk * kUTile; e += 256) {
      {  // e: row c, column i of the chunk (i fastest: contiguous in errs)
        const int c = e / kUChunk, i = e % kUChunk;
        es[i][c] = r0 + c < a.N ? a.errs[static_cast<size_t>(r0 + c) * kGroupCols + i0 + i] : 0.0;
      }
      {  // G: row i of the chunk, column c (c fastest: contiguous in G)
        const int c = e % kUTile, i = e / kUTile;
        gs[i][c] = j0 + c < a.K ? a.G[static_cast<size_t>(b0 + i0 + i) * a.K + j0 + c] : 0.0;
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int i = 0; i < kUChunk; ++i) {
      double ev[4], gv[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) ev[p] = es[i][ty * 4 + p];
#pragma unroll
      for (int q = 0; q < 4; ++q) gv[q] = gs[i][tx + 16 * q];
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = __dadd_rn(acc[p][q], __dmul_rn(ev[p], gv[q]));
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
      const int j = j0 + tx + 16 * q;
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
// Cholesky: for each block column kb, the diagonal tile is factored and its
// triangular inverse formed by one CTA, the panel below becomes
// L[ib][kb] = A[ib][kb] inv(L[kb][kb])^T, and the trailing lower triangle is
// updated, A[ib][jb] -= L[ib][kb] L[jb][kb]^T.  X = L^-1 follows by block rows
// one step behind (see the schedule below).  Every tile product is a
// 64 x 64 x 64 fp64 product: 256 threads, 4 x 4 outputs each (rows 4 tr + i,
// columns tc + 16 j), both operands staged row by row in shared memory.
constexpr int kB = 64;
constexpr int kBP = kB + 1;  // padded row (doubles): 16 rows read down one column hit 16 distinct bank pairs
constexpr int kFactorSmem = (2 * kB * kBP + kB + 32) * 8;

// dst[r][c] = src[r ld + c]: coalesced reads, consecutive shared-memory words.
__device__ __forceinline__ void stage_tile(double (*dst)[kBP], const double* src, long long ld) {
  for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) {
    const int r = e / kB, c = e % kB;
    dst[r][c] = src[static_cast<long long>(r) * ld + c];
  }
}

// acc[i][j] += sum_k P[4 tr + i][k] Q(k, tc + 16 j), with Q(k, c) = Qs[c][k] when
// QT (the staged tile is the transpose of the right operand), else Qs[k][c].  A
// warp reads two P addresses (broadcasts) and 16 consecutive, or column-wise
// conflict-free, Q words per load.
template <bool QT>
__device__ __forceinline__ void tile_product(double (&acc)[4][4], const double (*Ps)[kBP], const double (*Qs)[kBP],
                                             int tr, int tc) {
#pragma unroll 4
  for (int k = 0; k < kB; ++k) {
    double p[4], q[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      p[i] = Ps[4 * tr + i][k];
      q[i] = QT ? Qs[tc + 16 * i][k] : Qs[k][tc + 16 * i];
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fma(p[i], q[j], acc[i][j]);
  }
}

// Lower Cholesky factor of the 32 x 32 block at a[o..o+31][o..o+31], in place,
// by one warp, lane i keeping row o + i in registers: at column j every lane
// takes rs = 1/sqrt(a_jj) from lane j's register (a shuffle), L_jj = a_jj rs,
// lane i > j forms l_ij = a_ij rs and publishes it in col[i], and every lane
// updates its row, a_ic -= l_ij l_cj for j < c <= i (l_cj a broadcast read).
// rd[o + j] receives 1 / L_jj.  Entries above the diagonal become 0.
__device__ __forceinline__ void chol32_warp(double (*a)[kBP], double* col, double* rd, int o) {
  const int i = threadIdx.x & 31;
  double r[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) r[c] = c <= i ? a[o + i][o + c] : 0.0;
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const double ajj = __shfl_sync(0xffffffffu, r[j], j);
    const double rs = rsqrt(ajj);
    const double l = r[j] * rs;
    col[i] = l;
    __syncwarp();
#pragma unroll
    for (int c = j + 1; c < 32; ++c)
      if (i >= c) r[c] = fma(-l, col[c], r[c]);
    __syncwarp();  // col is rewritten for the next column
    if (i == j) {
      r[j] = ajj * rs;
      rd[o + j] = rs;
    } else if (i < j) {
      r[j] = 0.0;
    } else {
      r[j] = l;
    }
  }
#pragma unroll
  for (int c = 0; c < 32; ++c) a[o + i][o + c] = r[c];
}

// X = L^-1 for the lower-triangular 32 x 32 block L = a[o..][o..], into
// x[o..][o..], by one warp: lane c forms column c by forward substitution,
// X[i][c] = -(sum_{k<i} L[i][k] X[k][c]) / L[i][i] (X[k][c] = 0 for k < c, so the
// sum may start at 0), X[c][c] = 1 / L[c][c]; rd holds the 32 reciprocals.
// L is read by broadcasts, each lane's column of X is its own; two partial
// sums halve the dependent chain.
__device__ __forceinline__ void inv32_warp(const double (*a)[kBP], double (*x)[kBP], const double* rd, int o) {
  const int c = threadIdx.x & 31;
  for (int i = 0; i < 32; ++i) {
    double s0 = 0.0, s1 = 0.0;
    for (int k = 0; k + 1 < i; k += 2) {
      s0 = fma(a[o + i][o + k], x[o + k][o + c], s0);
      s1 = fma(a[o + i][o + k + 1], x[o + k + 1][o + c], s1);
    }
    if (i & 1) s0 = fma(a[o + i][o + i - 1], x[o + i - 1][o + c], s0);
    x[o + i][o + c] = i < c ? 0.0 : (i == c ? rd[o + i] : -(s0 + s1) * rd[o + i]);
  }
}

// Diagonal tile kb: L[kb][kb] (lower, zeros above) in place and Dinv[kb] = its
// inverse, by one CTA of 256 threads, as 2 x 2 blocks of 32: L11 = chol(A11),
// X11 = L11^-1, L21 = A21 X11^T, A22 -= L21 L21^T, L22 = chol(A22), X22 = L22^-1,
// X21 = -X22 (L21 X11).  The two Cholesky factors and inverses are single-warp
// steps; the four 32 x 32 products use every thread (4 outputs each).
__device__ void chol_diag_tile(double* sm, double* __restrict__ L, int K, int kb, double* __restrict__ Dinv) {
  double(*a)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*x)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  double* rd = sm + 2 * kB * kBP;  // 1 / L_jj
  double* col = rd + kB;             // a column of the 32 x 32 factor in progress
  double* tile = L + static_cast<long long>(kb) * kB * K + static_cast<long long>(kb) * kB;
  const int warp = threadIdx.x >> 5;
  const int pr = threadIdx.x >> 3, pc = threadIdx.x & 7;  // 32 rows x 8 threads, columns pc + 8 j
  __syncthreads();  // the shared memory may hold a tile product of this CTA
  stage_tile(a, tile, K);
  __syncthreads();
  if (warp == 0) {
    chol32_warp(a, col, rd, 0);
    __syncwarp();
    inv32_warp(a, x, rd, 0);
  }
  __syncthreads();
  {  // L21 = A21 X11^T (X11 is 0 above its diagonal)
    double s[4] = {};
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const double v = a[32 + pr][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) s[j] = fma(v, x[pc + 8 * j][k], s[j]);
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j) a[32 + pr][pc + 8 * j] = s[j];
  }
  __syncthreads();
  // A22 -= L21 L21^T on and below the diagonal
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c = pc + 8 * j;
    if (c <= pr) {
      double s = 0.0;
#pragma unroll 8
      for (int k = 0; k < 32; ++k) s = fma(a[32 + pr][k], a[32 + c][k], s);
      a[32 + pr][32 + c] -= s;
    }
  }
  __syncthreads();
  if (warp == 0) {
    chol32_warp(a, col, rd, 32);
    __syncwarp();
    inv32_warp(a, x, rd, 32);
  }
  __syncthreads();
  {  // T = L21 X11 into the unused upper-right block of x
    double s[4] = {};
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const double v = a[32 + pr][k];
#pragma unroll
      for (int j = 0; j < 4; ++j) s[j] = fma(v, x[k][pc + 8 * j], s[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) x[pr][32 + pc + 8 * j] = s[j];
  }
  __syncthreads();
  {  // X21 = -X22 T
    double s[4] = {};
#pragma unroll 8
    for (int k = 0; k < 32; ++k) {
      const double v = x[32 + pr][32 + k];
#pragma unroll
      for (int j = 0; j < 4; ++j) s[j] = fma(v, x[k][32 + pc + 8 * j], s[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) x[32 + pr][pc + 8 * j] = -s[j];
  }
  __syncthreads();
  double* dinv = Dinv + static_cast<long long>(kb) * kB * kB;
  for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) {
    const int r = e / kB, c = e % kB;
    tile[static_cast<long long>(r) * K + c] = c <= r ? a[r][c] : 0.0;
    dinv[e] = c <= r ? x[r][c] : 0.0;
  }
}

// Panel of block column kb, block row ib > kb: L[ib][kb] = A[ib][kb] Dinv[kb]^T.
__device__ void chol_panel_tile(double* sm, double* __restrict__ L, int K, int kb, int ib,
                                const double* __restrict__ Dinv) {
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  double* tile = L + static_cast<long long>(ib) * kB * K + static_cast<long long>(kb) * kB;
  stage_tile(Ps, tile, K);
  stage_tile(Qs, Dinv + static_cast<long long>(kb) * kB * kB, kB);
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product<true>(acc, Ps, Qs, tr, tc);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tile[static_cast<long long>(4 * tr + i) * K + tc + 16 * j] = acc[i][j];
}

// Trailing update after block column kb of tile (ib, jb), kb < jb <= ib:
// A[ib][jb] -= L[ib][kb] L[jb][kb]^T.
__device__ void chol_update_tile(double* sm, double* __restrict__ L, int K, int kb, int ib, int jb) {
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  stage_tile(Ps, L + static_cast<long long>(ib) * kB * K + static_cast<long long>(kb) * kB, K);
  stage_tile(Qs, L + static_cast<long long>(jb) * kB * K + static_cast<long long>(kb) * kB, K);
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product<true>(acc, Ps, Qs, tr, tc);
  double* tile = L + static_cast<long long>(ib) * kB * K + static_cast<long long>(jb) * kB;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double* d = tile + static_cast<long long>(4 * tr + i) * K + tc + 16 * j;
      *d -= acc[i][j];
    }
}

// X = L^-1 by right-looking forward substitution on block rows, X in place of
// the remaining right-hand side R (L X = I): at step jb, block row jb is final,
// X[jb][kb] = Dinv[jb] R[jb][kb] for kb < jb and X[jb][jb] = Dinv[jb]; then every
// later block row is updated, R[ib][kb] -= L[ib][jb] X[jb][kb] for kb <= jb < ib
// (R starts as the identity: its first update, at jb = kb, is a plain product).

// Tile kb <= jb of the final block row jb.
__device__ void trinv_final_tile(double* sm, int K, int jb, int kb, const double* __restrict__ Dinv,
                                 double* __restrict__ X) {
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  double* tile = X + static_cast<long long>(jb) * kB * K + static_cast<long long>(kb) * kB;
  const double* dinv = Dinv + static_cast<long long>(jb) * kB * kB;
  if (kb == jb) {
    for (int e = threadIdx.x; e < kB * kB; e += blockDim.x) tile[static_cast<long long>(e / kB) * K + e % kB] = dinv[e];
    return;
  }
  stage_tile(Ps, dinv, kB);
  stage_tile(Qs, tile, K);
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product<false>(acc, Ps, Qs, tr, tc);
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) tile[static_cast<long long>(4 * tr + i) * K + tc + 16 * j] = acc[i][j];
}

// Update after step jb of tile (ib, kb), kb <= jb < ib: R[ib][kb] -= L[ib][jb] X[jb][kb].
__device__ void trinv_update_tile(double* sm, const double* __restrict__ L, int K, int jb, int kb, int ib,
                                  double* __restrict__ X) {
  double(*Ps)[kBP] = reinterpret_cast<double(*)[kBP]>(sm);
  double(*Qs)[kBP] = reinterpret_cast<double(*)[kBP]>(sm + kB * kBP);
  stage_tile(Ps, L + static_cast<long long>(ib) * kB * K + static_cast<long long>(jb) * kB, K);
  stage_tile(Qs, X + static_cast<long long>(jb) * kB * K + static_cast<long long>(kb) * kB, K);
  __syncthreads();
  const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_product<false>(acc, Ps, Qs, tr, tc);
  double* tile = X + static_cast<long long>(ib) * kB * K + static_cast<long long>(kb) * kB;
  const bool first = kb == jb;  // R[ib][kb] is still the zero block of the identity
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      double* d = tile + static_cast<long long>(4 * tr + i) * K + tc + 16 * j;
      *d = first ? -acc[i][j] : *d - acc[i][j];
    }
}

// The schedule: two launches per block column s, the inverse one step behind
// the factorization, and the next diagonal tile factored by the CTA that
// applies its last update (so it overlaps the rest of that update):
//   launch A(s): the panel of block column s (nb - 1 - s CTAs) and the update
//                after block row s - 1 of X (s (nb - s) CTAs);
//   launch B(s): the trailing update after block column s (one CTA per tile of
//                the lower triangle; CTA 0 holds tile (s + 1, s + 1) and goes on
//                to factor it) and the final block row s of X (s + 1 CTAs).
// A(s) needs Dinv[s] and the updated block column s (from B(s - 1)), L's block
// column s - 1 (A(s - 1)) and X's block row s - 1 (B(s - 1)); B(s) needs the
// panel and the update of X's block row s (A(s)).  A diagonal tile 0 launch
// starts it.
__global__ void __launch_bounds__(256) gptq_factor_diag0_kernel(double* __restrict__ L, int K,
                                                                double* __restrict__ Dinv) {
  extern __shared__ double sm[];
  chol_diag_tile(sm, L, K, 0, Dinv);
}

__global__ void __launch_bounds__(256) gptq_factor_a_kernel(double* __restrict__ L, int K, int s, int nb,
                                                            const double* __restrict__ Dinv,
                                                            double* __restrict__ X) {
  extern __shared__ double sm[];
  const int m = nb - 1 - s;
  const int b = static_cast<int>(blockIdx.x);
  if (b < m) {
    chol_panel_tile(sm, L, K, s, s + 1 + b, Dinv);
    return;
  }
  const int e = b - m;  // over kb = 0 .. s - 1 (fastest), ib = s .. nb - 1
  trinv_update_tile(sm, L, K, s - 1, e % s, s + e / s, X);
}

__global__ void __launch_bounds__(256, 2) gptq_factor_b_kernel(double* __restrict__ L, int K, int s, int nb,
                                                            double* __restrict__ Dinv, double* __restrict__ X) {
  extern __shared__ double sm[];
  const int m = nb - 1 - s;
  const int nu = m * (m + 1) / 2;
  const int b = static_cast<int>(blockIdx.x);
  if (b < nu) {
    // b = t (t + 1) / 2 + c for tile row t, column c <= t of the trailing triangle
    int t = static_cast<int>((sqrt(8.0 * b + 1.0) - 1.0) / 2.0);
    while ((t + 1) * (t + 2) / 2 <= b) ++t;
    while (t * (t + 1) / 2 > b) --t;
    const int c = b - t * (t + 1) / 2;
    chol_update_tile(sm, L, K, s, s + 1 + t, s + 1 + c);
    if (b == 0) chol_diag_tile(sm, L, K, s + 1, Dinv);  // tile (s + 1, s + 1) took its last update
    return;
  }
  trinv_final_tile(sm, K, s, b - nu, Dinv, X);
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
  cudaError_t e = cudaSuccess;
  for (const void* f : {reinterpret_cast<const void*>(gptq_factor_diag0_kernel),
                        reinterpret_cast<const void*>(gptq_factor_a_kernel),
                        reinterpret_cast<const void*>(gptq_factor_b_kernel)})
    if (e == cudaSuccess) e = ensure_func_attr(f, cudaFuncAttributeMaxDynamicSharedMemorySize, kFactorSmem);
  if (e != cudaSuccess) return e;
  gptq_reverse_kernel<<<4 * device_sm_count(), 256, 0, st>>>(H, K, L);
  gptq_factor_diag0_kernel<<<1, 256, kFactorSmem, st>>>(L, K, Dinv);
  e = cudaGetLastError();
  for (int s = 0; s < nb && e == cudaSuccess; ++s) {
    const int m = nb - 1 - s;
    const int ga = m + s * (nb - s);
    if (ga > 0) gptq_factor_a_kernel<<<ga, 256, kFactorSmem, st>>>(L, K, s, nb, Dinv, X);
    gptq_factor_b_kernel<<<m * (m + 1) / 2 + s + 1, 256, kFactorSmem, st>>>(L, K, s, nb, Dinv, X);
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
