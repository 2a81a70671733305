// PCA calibration of the key basis on the GPU.
//
// The pages calibrate the rotation offline: P holds the principal directions
// of the keys of a calibration set ("Loki: Low-rank Keys for Efficient Sparse
// Attention", atlas.scime.ai summary, summary paragraph and section
// "Approach").  For every KV head g, with N calibration keys x_n:
//   mu  = (1/N) sum_n x_n
//   C   = (1/N) sum_n (x_n - mu)(x_n - mu)^T
//   C   = V diag(lambda) V^T,  P[:, j] = the eigenvector of the j-th largest
//         eigenvalue, its sign fixed so that its largest-magnitude entry is
//         positive.
// Everything is fp64; P is rounded to fp32 at the end.
//
// Three kernels: the means, the covariance (32x32 tiles of the upper
// triangle, one CTA each, fp64 accumulation in token order), and a cyclic
// Jacobi eigensolver with one CTA per head.  The eigensolver keeps the upper
// triangle of C (packed) and the accumulated rotations V in shared memory.
// Each round applies D/2 disjoint plane rotations chosen by the round-robin
// (circle) pairing, so that every pair (p, q) is met once per sweep of D-1
// rounds; a rotation (c, s) in plane (p, q) zeroes C[p][q].  The two-sided
// update of all rotations of a round is done block by block: the 2x2 block
// of C on the rows of pair i and the columns of pair j becomes
// R_i^T B R_j, R = [[c, s], [-s, c]], so no element is touched twice.
// Sweeps stop when the off-diagonal mass is below 1e-30 of the total (a
// relative off-diagonal norm of 1e-15) or after kPcaMaxSweeps sweeps.
#pragma once

#include "common.cuh"

namespace loki {

constexpr int kPcaThreads = 512;
constexpr int kPcaTile = 32;
constexpr int kPcaMaxSweeps = 30;

template <typename T>
struct PcaArgs {
  const T *keys;   // [H, N, D]
  int32_t n_heads;
  int32_t n_keys;
  double *mean;    // [H, D]
  double *cov;     // [H, D, D]; the kernels fill tiles with ti <= tj
};

struct PcaEigArgs {
  const double *cov;  // [H, D, D], upper triangle
  float *P;           // [H, D, D]
  double *eigvals;    // [H, D] or null
};

// mean[g][c]: grid (H, D/32), 256 threads; lane = column, warp = a stride of
// tokens, then the eight warps' partial sums in a fixed order.
template <typename T, int D>
__global__ void __launch_bounds__(256) pca_mean_kernel(const __grid_constant__ PcaArgs<T> a) {
  __shared__ double part[8][kPcaTile];
  const int g = blockIdx.x, c = blockIdx.y * kPcaTile + (threadIdx.x & 31), w = threadIdx.x >> 5;
  const T *x = a.keys + (size_t)g * a.n_keys * D + c;
  double s = 0.0;
  for (int n = w; n < a.n_keys; n += 8) s += (double)to_f32(x[(size_t)n * D]);
  part[w][threadIdx.x & 31] = s;
  __syncthreads();
  if (w == 0) {
    double t = 0.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) t += part[i][threadIdx.x];
    a.mean[(size_t)g * D + c] = t / (double)a.n_keys;
  }
}

// cov[g][32ti + i][32tj + j] for one upper tile (ti <= tj): grid (H, tiles),
// 256 threads, each owning four outputs (column i, rows 4 * (tid / 32) ..+4 of
// the tile's j).  Keys are staged 64 at a time, centred, in fp64.
template <typename T, int D>
__global__ void __launch_bounds__(256) pca_cov_kernel(const __grid_constant__ PcaArgs<T> a) {
  constexpr int NT = D / kPcaTile;
  constexpr int CH = 64;  // tokens per stage
  __shared__ double xs[CH][kPcaTile];
  __shared__ double ys[CH][kPcaTile];
  const int g = blockIdx.x;
  int ti = 0, rem = blockIdx.y;
  while (rem >= NT - ti) {
    rem -= NT - ti;
    ++ti;
  }
  const int tj = ti + rem;
  const int tid = threadIdx.x, i = tid & 31, j0 = 4 * (tid >> 5);
  const T *x = a.keys + (size_t)g * a.n_keys * D;
  const double *mu = a.mean + (size_t)g * D;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int n0 = 0; n0 < a.n_keys; n0 += CH) {
    __syncthreads();  // the previous stage is consumed
    for (int e = tid; e < CH * kPcaTile; e += 256) {
      const int r = e / kPcaTile, cc = e % kPcaTile, n = n0 + r;
      double xv = 0.0, yv = 0.0;
      if (n < a.n_keys) {
        xv = (double)to_f32(x[(size_t)n * D + ti * kPcaTile + cc]) - mu[ti * kPcaTile + cc];
        yv = (double)to_f32(x[(size_t)n * D + tj * kPcaTile + cc]) - mu[tj * kPcaTile + cc];
      }
      xs[r][cc] = xv;
      ys[r][cc] = yv;
    }
    __syncthreads();
    const int m = min(CH, a.n_keys - n0);
    for (int r = 0; r < m; ++r) {
      const double xv = xs[r][i];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fma(xv, ys[r][j0 + q], acc[q]);
    }
  }
  double *C = a.cov + (size_t)g * D * D;
#pragma unroll
  for (int q = 0; q < 4; ++q) C[(size_t)(ti * kPcaTile + i) * D + tj * kPcaTile + j0 + q] = acc[q] / (double)a.n_keys;
}

// Offset of element (x, y), x <= y, of a packed upper triangle of order D.
template <int D>
__device__ __forceinline__ int pk(int x, int y) {
  return x * D - (x * (x - 1)) / 2 + (y - x);
}

template <int D>
struct PcaSmem {
  static constexpr int kPacked = D * (D + 1) / 2;
  static constexpr int kA = 0;                       // doubles: packed upper triangle
  static constexpr int kV = kA + kPacked;            // doubles: V, row-major D x D
  static constexpr int kC = kV + D * D;              // doubles: c of each pair
  static constexpr int kS = kC + D / 2;              // doubles: s of each pair
  static constexpr int kT = kS + D / 2;              // doubles: t = s / c of each pair
  static constexpr int kRed = kT + D / 2;            // doubles: reduction scratch
  static constexpr int kDoubles = kRed + 2 * (kPcaThreads / 32);
  static constexpr int kPairs = kDoubles * 8;        // ints: p, q of each pair
  static constexpr int kBytes = kPairs + D * 4;
};

// The round-robin pairing of round r: position 0 holds index 0, positions
// 1 .. D-1 hold 1 + ((pos - 1 + r) mod (D - 1)); pair j joins positions j and
// D - 1 - j.
template <int D>
__device__ __forceinline__ void round_pair(int r, int j, int &p, int &q) {
  const int a = j == 0 ? 0 : 1 + ((j - 1 + r) % (D - 1));
  const int b = 1 + ((D - 2 - j + r) % (D - 1));
  p = min(a, b);
  q = max(a, b);
}

// Sum over the CTA of two doubles, returned to every thread.
__device__ __forceinline__ void pca_block_sum2(double &u, double &v, double *red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    u += __shfl_xor_sync(kFull, u, off);
    v += __shfl_xor_sync(kFull, v, off);
  }
  if (lane == 0) {
    red[2 * w] = u;
    red[2 * w + 1] = v;
  }
  __syncthreads();
  u = 0.0;
  v = 0.0;
  for (int i = 0; i < kPcaThreads / 32; ++i) {
    u += red[2 * i];
    v += red[2 * i + 1];
  }
  __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(kPcaThreads, 1) pca_jacobi_kernel(const __grid_constant__ PcaEigArgs a) {
  using L = PcaSmem<D>;
  constexpr int NP = D / 2;
  extern __shared__ __align__(16) double psm[];
  double *A = psm + L::kA;
  double *V = psm + L::kV;
  double *cs = psm + L::kC;
  double *sn = psm + L::kS;
  double *tn = psm + L::kT;
  double *red = psm + L::kRed;
  int *pq = reinterpret_cast<int *>(reinterpret_cast<unsigned char *>(psm) + L::kPairs);  // [NP][2]
  const int g = blockIdx.x, tid = threadIdx.x;
  const double *C = a.cov + (size_t)g * D * D;

  // the upper triangle of C (the covariance kernel wrote tiles with ti <= tj)
  for (int e = tid; e < D * D; e += kPcaThreads) {
    const int x = e / D, y = e % D;
    if (x <= y) A[pk<D>(x, y)] = C[(size_t)x * D + y];
    V[e] = x == y ? 1.0 : 0.0;
  }
  __syncthreads();

  for (int sweep = 0; sweep < kPcaMaxSweeps; ++sweep) {
    double off = 0.0, tot = 0.0;
    for (int e = tid; e < D * D; e += kPcaThreads) {
      const int x = e / D, y = e % D;
      if (x <= y) {
        const double v = A[pk<D>(x, y)];
        if (x == y)
          tot += v * v;
        else
          off += v * v;
      }
    }
    pca_block_sum2(off, tot, red);
    if (off <= 1e-30 * (tot + 2.0 * off)) break;  // uniform: every thread holds the same sums

    for (int r = 0; r < D - 1; ++r) {
      // the rotation of each pair: tan(phi) = t with t^2 + 2 theta t - 1 = 0,
      // theta = (a_qq - a_pp) / (2 a_pq), the smaller root
      if (tid < NP) {
        int p, q;
        round_pair<D>(r, tid, p, q);
        pq[2 * tid] = p;
        pq[2 * tid + 1] = q;
        const double apq = A[pk<D>(p, q)];
        double c = 1.0, s = 0.0, t = 0.0;
        if (apq != 0.0) {
          const double th = (A[pk<D>(q, q)] - A[pk<D>(p, p)]) / (2.0 * apq);
          const double ath = fabs(th);
          t = ath > 1e150 ? 0.5 / th : (th >= 0.0 ? 1.0 : -1.0) / (ath + sqrt(th * th + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          s = t * c;
        }
        cs[tid] = c;
        sn[tid] = s;
        tn[tid] = t;
      }
      __syncthreads();
      // C <- J^T C J block by block (upper triangle of blocks, i <= j)
      for (int e = tid; e < NP * NP; e += kPcaThreads) {
        const int i = e / NP, j = e % NP;
        if (j < i) continue;
        const int p = pq[2 * i], q = pq[2 * i + 1];
        if (i == j) {
          const int ipq = pk<D>(p, q);
          const double apq = A[ipq], t = tn[i];
          A[pk<D>(p, p)] -= t * apq;
          A[pk<D>(q, q)] += t * apq;
          A[ipq] = 0.0;
        } else {
          const int pp = pq[2 * j], qq = pq[2 * j + 1];
          const int i00 = pk<D>(min(p, pp), max(p, pp)), i01 = pk<D>(min(p, qq), max(p, qq));
          const int i10 = pk<D>(min(q, pp), max(q, pp)), i11 = pk<D>(min(q, qq), max(q, qq));
          const double b00 = A[i00], b01 = A[i01], b10 = A[i10], b11 = A[i11];
          const double ci = cs[i], si = sn[i], cj = cs[j], sj = sn[j];
          // rows: [c -s; s c] . B
          const double r00 = ci * b00 - si * b10, r01 = ci * b01 - si * b11;
          const double r10 = si * b00 + ci * b10, r11 = si * b01 + ci * b11;
          // columns: . [c s; -s c]
          A[i00] = r00 * cj - r01 * sj;
          A[i01] = r00 * sj + r01 * cj;
          A[i10] = r10 * cj - r11 * sj;
          A[i11] = r10 * sj + r11 * cj;
        }
      }
      // V <- V J: columns p, q of every row
      for (int e = tid; e < D * NP; e += kPcaThreads) {
        const int row = e / NP, j = e % NP;
        const int p = pq[2 * j], q = pq[2 * j + 1];
        const double c = cs[j], s = sn[j];
        const double vp = V[row * D + p], vq = V[row * D + q];
        V[row * D + p] = c * vp - s * vq;
        V[row * D + q] = s * vp + c * vq;
      }
      __syncthreads();
    }
  }

  // descending order (ties: lower index first), sign of each column, output
  if (tid < D) {
    const int x = tid;
    const double lx = A[pk<D>(x, x)];
    int rank = 0;
    for (int y = 0; y < D; ++y) {
      const double ly = A[pk<D>(y, y)];
      rank += (ly > lx || (ly == lx && y < x)) ? 1 : 0;
    }
    int lead = 0;
    double best = -1.0;
    for (int r = 0; r < D; ++r) {
      const double m = fabs(V[r * D + x]);
      if (m > best) {
        best = m;
        lead = r;
      }
    }
    const double sg = V[lead * D + x] < 0.0 ? -1.0 : 1.0;
    float *Pg = a.P + (size_t)g * D * D;
    for (int r = 0; r < D; ++r) Pg[(size_t)r * D + rank] = (float)(sg * V[r * D + x]);
    if (a.eigvals != nullptr) a.eigvals[(size_t)g * D + rank] = lx;
  }
}

}  // namespace loki
