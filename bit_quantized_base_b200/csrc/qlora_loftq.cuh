// qlora_loftq.cuh -- LoftQ initialisation of the adapter for a quantised base.
//
// "Training LLMs on a Budget: LoRA, QLoRA, and LoftQ", §4 "The algorithm: alternating
// quantization and SVD": minimise ||W - Q - s B A||_F by alternating Q = quantise(W - s B A) and
// s B A = the best rank-r approximation of R = W - Q (the top r singular triplets of R), starting
// from B A = 0; B = U_r sqrt(S_r / s), A = sqrt(S_r / s) V_r^T.  One iteration = one quantisation
// and one SVD.
//
// The top-r SVD of the [N, K] residual runs as randomized subspace iteration with Rayleigh-Ritz
// (Halko, Martinsson, Tropp, "Finding structure with randomness", 2011): a Rademacher test matrix
// of l = r + 16 columns, `power_iters` rounds of R R^T with the basis re-orthonormalised between
// products, then the small l x l eigenproblem of Z^T Z (Z = R^T Qb).  Every basis is made
// orthonormal by SVQB (Stathopoulos and Wu, 2002): X <- X P diag(lambda^-1/2) from the eigen-pairs
// of X^T X, columns whose lambda is below 1e-10 of the largest dropped (set to zero), twice; the
// power iteration's intermediate bases only need to stay well conditioned and take one shifted
// Cholesky QR step instead.
// The l x l symmetric eigenproblems are cyclic Jacobi (Golub and Van Loan, "Matrix
// Computations", §8.5) in fp64 in one CTA, with round-robin pairs so that l/2 rotations run at
// once.  The tall products are fp32 SIMT GEMMs (64 x 128 tiles, fixed-order split reductions);
// no step is randomised beyond the test matrix, so the result is bitwise reproducible.
#pragma once
#include "qlora_quant.cuh"

namespace qlora {
namespace loftq {
constexpr int kMaxL = 96;        // subspace width limit: two l x l fp64 matrices in shared memory
constexpr int kOversample = 16;
constexpr int kBM = 64, kBN = 128, kBK = 32;
constexpr int kJacobiThreads = 512;
constexpr int kJacobiMaxSweeps = 40;
constexpr int kNormBlocks = 592;
constexpr double kDropRel = 1e-10;   // SVQB / Ritz: eigenvalues below this share of the largest
__host__ __device__ constexpr int jacobi_pad(int l) { return (l + 1) & ~1; }
// Row stride L + 1 (odd): a warp walking down a column of doubles touches distinct banks.
__host__ __device__ constexpr size_t chol_smem(int l) { return size_t(l) * (l + 1) * sizeof(double); }
__host__ __device__ constexpr size_t jacobi_smem(int l) {
  return size_t(2) * jacobi_pad(l) * (jacobi_pad(l) + 1) * sizeof(double);
}
// Converged when the off-diagonal Frobenius norm is below 1e-12 of the diagonal's.
constexpr double kJacobiTol2 = 1e-24;
}  // namespace loftq

// C[z][m][n] = sum over k in chunk z of opA(m, k) opB(k, n); chunk z = [z kchunk, (z+1) kchunk)
// clipped to Kk.  opA(m, k) = TA ? A[k lda + m] : A[m lda + k]; opB(k, n) = TB ? B[n ldb + k]
// : B[k ldb + n].  256 threads, a 64 x 128 tile, each thread 4 rows x 8 columns strided by 16 so
// that a warp's shared-memory reads fall in distinct banks; the next 32-deep slice is fetched
// into registers while the current one is multiplied.
template <bool TA, bool TB>
__global__ void __launch_bounds__(256)
loftq_gemm_kernel(const float* __restrict__ A, int64_t lda, const float* __restrict__ B,
                  int64_t ldb, float* __restrict__ C, int64_t ldc, int64_t zstride, int M, int Nn,
                  int64_t Kk, int64_t kchunk) {
  using namespace loftq;
  constexpr int kAPer = kBM * kBK / 256, kBPer = kBK * kBN / 256;
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN;
  const int64_t kbeg = int64_t(blockIdx.z) * kchunk;
  const int64_t kend = kbeg + kchunk < Kk ? kbeg + kchunk : Kk;
  float ra[kAPer], rb[kBPer];
  auto fetch = [&](int64_t k0) {
#pragma unroll
    for (int t = 0; t < kAPer; ++t) {
      const int i = threadIdx.x + 256 * t;
      const int mm = TA ? i % kBM : i / kBK;
      const int kk = TA ? i / kBM : i % kBK;
      const int m = m0 + mm;
      const int64_t k = k0 + kk;
      ra[t] = (m < M && k < kend) ? (TA ? A[k * lda + m] : A[int64_t(m) * lda + k]) : 0.0f;
    }
#pragma unroll
    for (int t = 0; t < kBPer; ++t) {
      const int i = threadIdx.x + 256 * t;
      const int nn = TB ? i / kBK : i % kBN;
      const int kk = TB ? i % kBK : i / kBN;
      const int n = n0 + nn;
      const int64_t k = k0 + kk;
      rb[t] = (n < Nn && k < kend) ? (TB ? B[int64_t(n) * ldb + k] : B[k * ldb + n]) : 0.0f;
    }
  };
  float acc[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  if (kbeg < kend) fetch(kbeg);
  for (int64_t k0 = kbeg; k0 < kend; k0 += kBK) {
#pragma unroll
    for (int t = 0; t < kAPer; ++t) {
      const int i = threadIdx.x + 256 * t;
      As[TA ? i / kBM : i % kBK][TA ? i % kBM : i / kBK] = ra[t];
    }
#pragma unroll
    for (int t = 0; t < kBPer; ++t) {
      const int i = threadIdx.x + 256 * t;
      Bs[TB ? i % kBK : i / kBN][TB ? i / kBK : i % kBN] = rb[t];
    }
    __syncthreads();
    if (k0 + kBK < kend) fetch(k0 + kBK);
#pragma unroll
    for (int kk = 0; kk < kBK; ++kk) {
      float a[4], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 8; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* Cz = C + int64_t(blockIdx.z) * zstride;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n < Nn) Cz[int64_t(m) * ldc + n] = acc[i][j];
    }
  }
}

// out[i] = sum over z = 0..Z-1 in order of part[z zstride + i] (binary64), stored as fp32 or fp64.
__global__ void __launch_bounds__(256)
loftq_reduce_kernel(const float* __restrict__ part, int64_t zstride, int Z, int64_t count,
                    float* out32, double* out64) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += int64_t(gridDim.x) * blockDim.x) {
    double s = 0.0;
    for (int z = 0; z < Z; ++z) s += double(part[int64_t(z) * zstride + i]);
    if (out64) out64[i] = s;
    else out32[i] = float(s);
  }
}

// Rademacher test matrix: entry i = +-1 from bit 63 of the SplitMix64 output for seed + i
// (Steele, Lea, Flood, "Fast splittable pseudorandom number generators", 2014).
__global__ void loftq_omega_kernel(float* omega, int64_t count, uint64_t seed) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += int64_t(gridDim.x) * blockDim.x) {
    uint64_t z = seed + uint64_t(i + 1) * 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    z ^= z >> 31;
    omega[i] = (z >> 63) ? 1.0f : -1.0f;
  }
}

struct JacobiParams {
  const double* G;   // [l, l] symmetric
  int l;
  int mode;          // 0: SVQB transform M [l, l]; 1: Ritz factors Cb [l, r], Ca [r, l], sigma [r]
  float* M;
  float* Cb;
  float* Ca;
  float* sigma;
  int r;
  float s;
  int* sweeps;       // optional: sweeps used (diagnostics)
};

__device__ __forceinline__ double block_sum_jacobi(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double s = 0.0;
  for (int w = 0; w < int(blockDim.x >> 5); ++w) s += red[w];
  return s;
}

// Eigen-decomposition G = P diag(lambda) P^T by cyclic Jacobi, fp64, one CTA.  Round-robin
// ("circle") ordering: in round t of L - 1, index 0 stays and the others rotate, pairing
// pos(k) with pos(L-1-k); the L/2 rotations of a round touch disjoint rows and columns, so they
// are applied together: first to the columns of G and P (G J, P J), then to the rows (J^T G).
__global__ void __launch_bounds__(loftq::kJacobiThreads) loftq_jacobi_kernel(const JacobiParams p) {
  using namespace loftq;
  extern __shared__ double jsm[];
  const int l = p.l, L = jacobi_pad(l), S = L + 1;
  double* a = jsm;              // [L, S]
  double* v = jsm + L * S;      // [L, S]
  __shared__ double cs[kMaxL / 2], sn[kMaxL / 2];
  __shared__ int pp[kMaxL / 2], qq[kMaxL / 2];
  __shared__ double red[kJacobiThreads / 32];
  __shared__ int order[kMaxL];
  __shared__ int done;
  for (int i = threadIdx.x; i < L * L; i += blockDim.x) {
    const int r = i / L, c = i % L;
    a[r * S + c] = (r < l && c < l) ? p.G[r * l + c] : 0.0;
    v[r * S + c] = r == c ? 1.0 : 0.0;
  }
  __syncthreads();
  int sweep = 0;
  for (; sweep < kJacobiMaxSweeps; ++sweep) {
    double off = 0.0, dia = 0.0;
    for (int i = threadIdx.x; i < L * L; i += blockDim.x) {
      const int r = i / L, c = i % L;
      const double x = a[r * S + c] * a[r * S + c];
      if (r == c) dia += x;
      else off += x;
    }
    off = block_sum_jacobi(off, red);
    dia = block_sum_jacobi(dia, red);
    if (threadIdx.x == 0) done = !(off > kJacobiTol2 * dia);
    __syncthreads();
    if (done) break;
    for (int t = 0; t < L - 1; ++t) {
      if (threadIdx.x < L / 2) {
        const int k = threadIdx.x;
        const int i0 = k, i1 = L - 1 - k;
        const int P0 = i0 == 0 ? 0 : 1 + (i0 - 1 + t) % (L - 1);
        const int P1 = 1 + (i1 - 1 + t) % (L - 1);
        const int P = P0 < P1 ? P0 : P1, Q = P0 < P1 ? P1 : P0;
        const double apq = a[P * S + Q];
        double c = 1.0, s = 0.0;
        if (apq != 0.0) {
          const double tau = (a[Q * S + Q] - a[P * S + P]) / (2.0 * apq);
          const double tt = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
          c = rsqrt(1.0 + tt * tt);
          s = tt * c;
        }
        cs[k] = c;
        sn[k] = s;
        pp[k] = P;
        qq[k] = Q;
      }
      __syncthreads();
      for (int i = threadIdx.x; i < L * (L / 2); i += blockDim.x) {   // columns: G J, P J
        const int row = i % L, k = i / L;
        const double c = cs[k], s = sn[k];
        const int P = pp[k], Q = qq[k];
        const double x = a[row * S + P], y = a[row * S + Q];
        a[row * S + P] = c * x - s * y;
        a[row * S + Q] = s * x + c * y;
        const double vx = v[row * S + P], vy = v[row * S + Q];
        v[row * S + P] = c * vx - s * vy;
        v[row * S + Q] = s * vx + c * vy;
      }
      __syncthreads();
      for (int i = threadIdx.x; i < L * (L / 2); i += blockDim.x) {   // rows: J^T (G J)
        const int col = i % L, k = i / L;
        const double c = cs[k], s = sn[k];
        const int P = pp[k], Q = qq[k];
        const double x = a[P * S + col], y = a[Q * S + col];
        a[P * S + col] = c * x - s * y;
        a[Q * S + col] = s * x + c * y;
      }
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) {
    if (p.sweeps) *p.sweeps = sweep;
    for (int i = 0; i < l; ++i) order[i] = i;          // descending eigenvalues, stable
    for (int i = 1; i < l; ++i) {
      const int o = order[i];
      const double key = a[o * S + o];
      int j = i - 1;
      while (j >= 0 && a[order[j] * S + order[j]] < key) {
        order[j + 1] = order[j];
        --j;
      }
      order[j + 1] = o;
    }
  }
  __syncthreads();
  const double lmax = fmax(a[order[0] * S + order[0]], 0.0);
  if (p.mode == 0) {
    for (int i = threadIdx.x; i < l * l; i += blockDim.x) {
      const int row = i / l, j = i % l;
      const double lam = a[j * S + j];
      const double sc = lam > kDropRel * lmax && lam > 0.0 ? 1.0 / sqrt(lam) : 0.0;
      p.M[row * l + j] = float(v[row * S + j] * sc);
    }
  } else {
    const double smax = sqrt(lmax);
    for (int i = threadIdx.x; i < l * p.r; i += blockDim.x) {
      const int row = i / p.r, j = i % p.r;
      const int e = order[j];
      const double sig = sqrt(fmax(a[e * S + e], 0.0));
      const bool keep = sig > 0.0 && sig * sig > kDropRel * smax * smax;
      const double x = v[row * S + e];
      p.Cb[row * p.r + j] = keep ? float(x * sqrt(sig / double(p.s))) : 0.0f;
      p.Ca[j * l + row] = keep ? float(x / sqrt(double(p.s) * sig)) : 0.0f;
      if (row == 0) p.sigma[j] = float(sig);
    }
  }
}

// Shifted Cholesky QR step for the power iteration's intermediate bases (Fukaya, Kannan,
// Nakatsukasa, Yamamoto, Yanagisawa, "Shifted Cholesky QR for computing the QR factorization of
// ill-conditioned matrices", 2020): G + delta I = L L^T with delta = 1e-5 of G's largest
// diagonal entry, M = L^-T, so that X M has nearly orthonormal columns; directions of X whose
// energy is below delta come out damped, which an intermediate basis can afford (the basis that
// Rayleigh-Ritz uses is made by SVQB).  A pivot that the shift does not keep positive drops its
// column (M's column zero); an all-zero G gives M = 0.  fp64, one CTA: the factorisation is
// column by column, then each thread solves L x = e_c for one column c.
__global__ void __launch_bounds__(loftq::kJacobiThreads) loftq_chol_kernel(const double* G, int l,
                                                                          float* M) {
  using namespace loftq;
  extern __shared__ double csm[];
  const int S = l + 1;                    // padded stride: column walks spread over banks
  double* Lm = csm;                       // [l, S], lower triangle
  __shared__ double delta;
  __shared__ int dropped[kMaxL];
  for (int i = threadIdx.x; i < l * l; i += blockDim.x) Lm[(i / l) * S + i % l] = G[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    double dmax = 0.0;
    for (int i = 0; i < l; ++i) dmax = fmax(dmax, Lm[i * S + i]);
    delta = 1e-5 * dmax;
  }
  __syncthreads();
  if (!(delta > 0.0)) {
    for (int i = threadIdx.x; i < l * l; i += blockDim.x) M[i] = 0.0f;
    return;
  }
  for (int i = threadIdx.x; i < l; i += blockDim.x) Lm[i * S + i] += delta;
  __syncthreads();
  for (int j = 0; j < l; ++j) {
    const double d = Lm[j * S + j];
    const bool drop = !(d > 0.5 * delta);
    const double piv = drop ? 0.0 : sqrt(d);
    __syncthreads();
    if (threadIdx.x == 0) {
      dropped[j] = drop;
      Lm[j * S + j] = drop ? 1.0 : piv;
    }
    for (int i = j + 1 + threadIdx.x; i < l; i += blockDim.x)
      Lm[i * S + j] = drop ? 0.0 : Lm[i * S + j] / piv;
    __syncthreads();
    const int m = l - j - 1;              // trailing update of the lower triangle
    for (int t = threadIdx.x; t < m * m; t += blockDim.x) {
      const int i = j + 1 + t / m, k = j + 1 + t % m;
      if (k <= i) Lm[i * S + k] -= Lm[i * S + j] * Lm[k * S + j];
    }
    __syncthreads();
  }
  // column c of L^-1 by forward substitution; M = L^-T, i.e. M[i][c] = (L^-1)[c][i]
  for (int c = threadIdx.x; c < l; c += blockDim.x) {
    double x[kMaxL];
    for (int i = 0; i < l; ++i) {
      if (i < c || dropped[i]) {
        x[i] = 0.0;
        continue;
      }
      double acc = i == c ? 1.0 : 0.0;
      for (int k = c; k < i; ++k) acc -= Lm[i * S + k] * x[k];
      x[i] = acc / Lm[i * S + i];
    }
    for (int i = 0; i < l; ++i) M[c * l + i] = float(x[i]);
  }
}

// R = W - deq(Q) (fp32) with per-CTA partial sums of R^2 (binary64, fixed element assignment).
template <int FMT>
__global__ void __launch_bounds__(256)
loftq_residual_kernel(const float* __restrict__ W, const StoredView q, float* __restrict__ R,
                      int N, int K, double* __restrict__ part) {
  __shared__ double red[8];
  const int64_t total = int64_t(N) * K;
  double acc = 0.0;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int n = int(i / K), k = int(i % K);
    const float x = W[i] - decode_element<FMT>(q, n, k);
    R[i] = x;
    acc += double(x) * double(x);
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < 8; ++w) s += red[w];
    part[blockIdx.x] = s;
  }
}

// With L = s Bf Af (fp32, the r-term sum in order): partial sums of (R - L)^2, and when write_v
// the quantiser's next input V = W - L written over R.  Each thread takes 4 consecutive elements
// of a row (K % 64 == 0), so one float4 of Af serves 4 outputs.
__global__ void __launch_bounds__(256)
loftq_shift_kernel(const float* __restrict__ W, float* RV, const float* __restrict__ Bf,
                   const float* __restrict__ Af, int N, int K, int r, float s, int write_v,
                   double* __restrict__ part) {
  __shared__ double red[8];
  const int64_t total4 = int64_t(N) * K / 4;
  double acc = 0.0;
  for (int64_t i4 = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i4 < total4;
       i4 += int64_t(gridDim.x) * blockDim.x) {
    const int64_t i = i4 * 4;
    const int n = int(i / K), k = int(i % K);
    float4 lr = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    const float* brow = Bf + int64_t(n) * r;
    for (int j = 0; j < r; ++j) {
      const float b = brow[j];
      const float4 av = *reinterpret_cast<const float4*>(Af + int64_t(j) * K + k);
      lr.x = fmaf(b, av.x, lr.x);
      lr.y = fmaf(b, av.y, lr.y);
      lr.z = fmaf(b, av.z, lr.z);
      lr.w = fmaf(b, av.w, lr.w);
    }
    lr.x *= s;
    lr.y *= s;
    lr.z *= s;
    lr.w *= s;
    const float4 rv = *reinterpret_cast<const float4*>(RV + i);
    const float ex = rv.x - lr.x, ey = rv.y - lr.y, ez = rv.z - lr.z, ew = rv.w - lr.w;
    acc += double(ex) * double(ex) + double(ey) * double(ey) + double(ez) * double(ez) +
           double(ew) * double(ew);
    if (write_v) {
      const float4 w = *reinterpret_cast<const float4*>(W + i);
      *reinterpret_cast<float4*>(RV + i) = make_float4(w.x - lr.x, w.y - lr.y, w.z - lr.z, w.w - lr.w);
    }
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    part[blockIdx.x] = t;
  }
}

// out = sqrt(sum of the partials, in order).
__global__ void loftq_norm_kernel(const double* part, int n, float* out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += part[i];
  *out = float(sqrt(s));
}

// fp32 -> bf16 (round to nearest even).
__global__ void loftq_to_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                     int64_t count) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += int64_t(gridDim.x) * blockDim.x)
    y[i] = __float2bfloat16_rn(x[i]);
}

}  // namespace qlora
