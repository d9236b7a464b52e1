// cluster.cu -- per-head bidirectional QK co-clustering (SVOO abstract; iCATS
// sections 3.1 and 4.1): k-means of the query tokens and of the key tokens,
// each side's distance being the interaction error under the metric of the
// other side's clusters, M = sum_b n_b c_b c_b^T / sum_b n_b (identity in the
// cold first query step).
//
// Kernels of one half-step (one side):
//   metric_m_kernel      M from the other side's centroids and sizes (fp64)
//   metric_nu_kernel     nu_j = M mu_j, kappa_j = mu_j . nu_j (fp64), |nu_j|, bf16(nu_j)
//   assign_update_kernel tcgen05 bf16 MMA of a 128-token tile against all
//                        bf16(nu_j) into TMEM; per token the score
//                        kappa_j - 2 x.nu_j is bounded by the MMA error, every
//                        candidate that can still win is re-evaluated in fp64
//                        and the argmin (ties to the smaller j) is the label;
//                        then the tile's tokens are sorted by label and each
//                        label run is summed in fp64 and added atomically
//                        (exact, so order-independent).
//   finalize_kernel      centroid = fp32(sum / count), empty clusters keep
//                        theirs; resets the sums for the next half-step.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace svoo {


// ---------------------------------------------------------------- init

__global__ void init_centroids_kernel(const uint16_t* __restrict__ x, int N, int nv, int d, int C,
                                      float* __restrict__ cent) {
  int h = blockIdx.y, j = blockIdx.x;
  long long idx = static_cast<long long>(j) * nv / C;
  const uint16_t* row = x + (static_cast<size_t>(h) * N + idx) * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x)
    cent[(static_cast<size_t>(h) * C + j) * d + i] = bf16_to_f32(row[i]);
}

// ---------------------------------------------------------------- metric

// M[h] = sum_b n_b c_b c_b^T / sum_b n_b in fp64. grid (T*(T+1)/2, BH) with
// T = d/16 output tiles per side (upper triangle only; each tile is written
// to both (i, j) and (j, i), so M is exactly symmetric), block 256 = 16 x 16,
// one output per thread; clusters staged 64 at a time.
constexpr int kMetricChunk = 64;

__global__ void __launch_bounds__(256)
    metric_m_kernel(const float* __restrict__ cent, const int32_t* __restrict__ sizes, int C, int d,
                    double* __restrict__ M) {
  __shared__ double ci[kMetricChunk][17];
  __shared__ double cj[kMetricChunk][17];
  const int h = blockIdx.y, T = d / 16;
  int t = blockIdx.x, ti = 0;
  while (t >= T - ti) {  // upper-triangle tile index -> (ti, tj), ti <= tj
    t -= T - ti;
    ++ti;
  }
  const int tj = ti + t;
  const int a = threadIdx.x >> 4, b = threadIdx.x & 15;
  const int i0 = ti * 16, j0 = tj * 16;
  double acc = 0.0;
  long long total = 0;
  for (int b0 = 0; b0 < C; b0 += kMetricChunk) {
    const int nb = min(kMetricChunk, C - b0);
    __syncthreads();
    for (int e = threadIdx.x; e < nb * 16; e += blockDim.x) {
      const int bb = e >> 4, c = e & 15;
      const float* cb = cent + (static_cast<size_t>(h) * C + b0 + bb) * d;
      const double n = static_cast<double>(sizes[h * C + b0 + bb]);
      ci[bb][c] = n * static_cast<double>(cb[i0 + c]);
      cj[bb][c] = static_cast<double>(cb[j0 + c]);
    }
    __syncthreads();
    for (int bb = 0; bb < nb; ++bb) acc = fma(ci[bb][a], cj[bb][b], acc);
  }
  for (int bb = 0; bb < C; ++bb) total += sizes[h * C + bb];
  const double v = total > 0 ? acc / static_cast<double>(total) : ((i0 + a) == (j0 + b) ? 1.0 : 0.0);
  double* Mh = M + static_cast<size_t>(h) * d * d;
  Mh[static_cast<size_t>(i0 + a) * d + j0 + b] = v;
  if (ti != tj) Mh[static_cast<size_t>(j0 + b) * d + i0 + a] = v;
}

// nu_j = M mu_j, kappa_j = mu_j . nu_j (fp64), bf16(nu_j), fp32 kappa and |nu_j|;
// clusters j in [C, Cpad) are padding (nu = 0, kappa = +inf). grid (Cpad/32, BH),
// block 256: warp w owns clusters j0 + 4w .. +3, lane owns dimensions 4 lane .. +3
// (d = 128; for d = 64 lanes 16..31 idle). M == nullptr means identity.
__global__ void __launch_bounds__(256)
    metric_nu_kernel(const double* __restrict__ M, const float* __restrict__ cent, int C, int Cpad,
                     int d, double* __restrict__ nu64, uint16_t* __restrict__ nu_bf16,
                     double* __restrict__ kappa64, float* __restrict__ kappa32,
                     float* __restrict__ nunorm) {
  __shared__ float mu[32][129];      // this block's 32 clusters, all dimensions (exact fp32)
  __shared__ double mch[16][128];    // 16 rows of M
  const int h = blockIdx.y, j0 = blockIdx.x * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e < 32 * d; e += blockDim.x) {
    const int r = e / d, c = e % d;
    mu[r][c] = (j0 + r < C) ? cent[(static_cast<size_t>(h) * C + j0 + r) * d + c] : 0.f;
  }
  const bool live = 4 * lane < d;
  double acc[4][4];  // [cluster][dimension]
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.0;
  if (M) {
    const double* Mh = M + static_cast<size_t>(h) * d * d;
    for (int l0 = 0; l0 < d; l0 += 16) {
      __syncthreads();
      for (int e = threadIdx.x; e < 16 * d; e += blockDim.x) mch[e / d][e % d] = Mh[static_cast<size_t>(l0) * d + e];
      __syncthreads();
      if (live) {
        for (int l = 0; l < 16; ++l) {
          // M symmetric: nu_j[i] = sum_l M[l][i] mu_j[l]
          const double2 m01 = *reinterpret_cast<const double2*>(&mch[l][4 * lane]);
          const double2 m23 = *reinterpret_cast<const double2*>(&mch[l][4 * lane + 2]);
          const double mv[4] = {m01.x, m01.y, m23.x, m23.y};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const double m_u = static_cast<double>(mu[4 * warp + u][l0 + l]);
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[u][v] = fma(mv[v], m_u, acc[u][v]);
          }
        }
      }
    }
  } else {
    __syncthreads();
    if (live)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = static_cast<double>(mu[4 * warp + u][4 * lane + v]);
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = j0 + 4 * warp + u;
    double k1 = 0.0, k2 = 0.0;
    if (live) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int i = 4 * lane + v;
        k1 = fma(static_cast<double>(mu[4 * warp + u][i]), acc[u][v], k1);
        k2 = fma(acc[u][v], acc[u][v], k2);
        if (j < C) nu64[(static_cast<size_t>(h) * C + j) * d + i] = acc[u][v];
        __nv_bfloat16 bv = __float2bfloat16_rn(j < C ? static_cast<float>(acc[u][v]) : 0.f);
        nu_bf16[(static_cast<size_t>(h) * Cpad + j) * d + i] = *reinterpret_cast<uint16_t*>(&bv);
      }
    }
    for (int o = 16; o > 0; o >>= 1) {
      k1 += __shfl_xor_sync(0xffffffffu, k1, o);
      k2 += __shfl_xor_sync(0xffffffffu, k2, o);
    }
    if (lane == 0) {
      kappa64[h * Cpad + j] = j < C ? k1 : INFINITY;
      kappa32[h * Cpad + j] = j < C ? static_cast<float>(k1) : INFINITY;
      nunorm[h * Cpad + j] = j < C ? static_cast<float>(sqrt(k2)) : 0.f;
    }
  }
}

// ---------------------------------------------------------------- assign + update
//
// One CTA (256 threads) walks `tiles_per_cta` tiles of 128 tokens of one head.
// Per tile: TMA load of X (128B-swizzled K-major), one tcgen05 MMA chain
// X . bf16(nu)^T into TMEM (128 lanes x Cpad fp32 columns). Thread (r, h)
// (warps w and w + 4 share TMEM lanes 32(w % 4).., h = w / 4) owns half h of
// row r's scores s_j = kappa_j - 2 x.nu_j. Pass 1 finds the half's minimum;
// with the row minimum m and the MMA error bound E, pass 2 lists the columns
// with s_j <= m + 2E (they contain the exact argmin). A row with a single
// candidate takes it; otherwise one warp re-scores its candidates in fp64
// (kappa_j - 2 x.nu_j, dimensions split over the lanes) and the minimum wins,
// ties to the smaller j. The tile's tokens are then grouped by label (counting
// sort in shared memory) and each label run of each (4-dimension group, slice)
// is summed in fp64 and added to the head's sums with one atomic per run.

constexpr int kAssignThreads = 256;
constexpr int kTileRows = 128;
constexpr int kSlots = 8;  // candidate slots per half-row; more -> full re-score

struct AssignSmem {
  int abort;
  uint32_t tmem_base;
  uint64_t tma_bar;
  uint64_t mma_bar;
  float max_nrm;
  float max_kap;
  int namb;
  float xn2[2][kTileRows];
  float mh[2][kTileRows];
  int kc[2][kTileRows];                 // candidates per half (kSlots + 1 = overflow)
  int16_t slot[kTileRows][2][kSlots];
  int lab[kTileRows];
  int pos[kTileRows];
  int16_t amb[kTileRows];
  int16_t sorted_row[kTileRows];
  int16_t sorted_lab[kTileRows];
  int lstart[256];
  int wsum[8];
  float red[8];
};
constexpr int kAssignHeader = 12288;  // AssignSmem + per-CTA counts, keeps the X tile 1024-aligned
static_assert(sizeof(AssignSmem) + 256 * sizeof(int) <= kAssignHeader, "header overflow");

// bf16 pair (columns c, c+1, c even) of row `row` in a 128-row swizzled X tile
__device__ __forceinline__ uint32_t x_pair(const uint8_t* xs, int row, int c) {
  return *reinterpret_cast<const uint32_t*>(xs + sw128_offset(row, c, kTileRows));
}

// fp64 score kappa_j - 2 x_row . nu_j, computed by the whole warp (lane = 2 or 4 dims)
__device__ __forceinline__ double warp_score(const uint8_t* xs, int row, const double* nj, double kap,
                                             int d, int lane) {
  double part = 0.0;
  for (int c = lane * 2; c < d; c += 64) {
    const uint32_t xp = x_pair(xs, row, c);
    const double2 n2 = *reinterpret_cast<const double2*>(nj + c);
    part = fma(static_cast<double>(__uint_as_float(xp << 16)), n2.x, part);
    part = fma(static_cast<double>(__uint_as_float(xp & 0xffff0000u)), n2.y, part);
  }
  for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  return kap - 2.0 * part;
}

// grid (ceil(ntiles / tiles_per_cta), BH), block 256.
// Dynamic smem: [AssignSmem + counts, 12 KB][X tile 128 x d bf16][nu Cpad x d bf16][kappa][nunorm]
__global__ void __launch_bounds__(kAssignThreads, 2)
    assign_update_kernel(const __grid_constant__ CUtensorMap xmap, int N, int nv, int d, int C,
                         int Cpad, int tmem_cols, int tiles_per_cta,
                         const uint16_t* __restrict__ nu_bf16, const double* __restrict__ nu64,
                         const double* __restrict__ kappa64, const float* __restrict__ kappa_g,
                         const float* __restrict__ nunorm_g, int32_t* __restrict__ assign,
                         double* __restrict__ sums, int32_t* __restrict__ counts,
                         int* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AssignSmem* S = reinterpret_cast<AssignSmem*>(base);
  int* cnt = reinterpret_cast<int*>(base + sizeof(AssignSmem));
  uint8_t* xs = base + kAssignHeader;
  uint8_t* nus = xs + kTileRows * d * 2;
  float* kap = reinterpret_cast<float*>(nus + static_cast<size_t>(Cpad) * d * 2);
  float* nrm = kap + Cpad;

  const int h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = (nv + kTileRows - 1) / kTileRows;
  const int t_begin = blockIdx.x * tiles_per_cta;
  const int t_end = min(ntiles, t_begin + tiles_per_cta);
  if (t_begin >= t_end || timed_out_before(err)) return;

  if (tid == 0) {
    S->abort = 0;
    mbar_init(smem_u32(&S->tma_bar), 1);
    mbar_init(smem_u32(&S->mma_bar), 1);
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
  }
  __syncwarp();
  if (warp == 0) {
    tmem_alloc(smem_u32(&S->tmem_base), tmem_cols);
    tmem_relinquish();
  }
  // nu (bf16) into the 128B-swizzled K-major layout the MMA expects; kappa, |nu|
  {
    const int chunks = d / 8;
    const uint4* src = reinterpret_cast<const uint4*>(nu_bf16 + static_cast<size_t>(h) * Cpad * d);
    for (int e = tid; e < Cpad * chunks; e += blockDim.x) {
      int j = e / chunks, c = e % chunks;
      *reinterpret_cast<uint4*>(nus + sw128_offset(j, c * 8, Cpad)) = src[e];
    }
    float mn = 0.f, mk = 0.f;
    for (int j = tid; j < Cpad; j += blockDim.x) {
      kap[j] = kappa_g[h * Cpad + j];
      nrm[j] = nunorm_g[h * Cpad + j];
      cnt[j] = 0;
      mn = fmaxf(mn, nrm[j]);
      if (j < C) mk = fmaxf(mk, fabsf(kap[j]));
    }
    for (int o = 16; o > 0; o >>= 1) {
      mn = fmaxf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
    }
    if (lane == 0) S->red[warp] = mn;
    __syncthreads();
    if (tid == 0) {
      float a = 0.f;
      for (int w = 0; w < 8; ++w) a = fmaxf(a, S->red[w]);
      S->max_nrm = a;
    }
    __syncthreads();
    if (lane == 0) S->red[warp] = mk;
    __syncthreads();
    if (tid == 0) {
      float a = 0.f;
      for (int w = 0; w < 8; ++w) a = fmaxf(a, S->red[w]);
      S->max_kap = a;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;
  volatile int* abort = &S->abort;

  const uint32_t idesc = idesc_bf16_f32(128, Cpad, false, false);
  const uint32_t xs_u32 = smem_u32(xs), nus_u32 = smem_u32(nus);
  const double* nu_h = nu64 + static_cast<size_t>(h) * C * d;
  const double* kap64 = kappa64 + static_cast<size_t>(h) * Cpad;
  const size_t xrow0 = static_cast<size_t>(h) * N;
  const int r = ((warp & 3) << 5) | lane;  // token row == TMEM lane
  const int half = warp >> 2;
  const int ncol = Cpad / 2;               // columns of this thread's half
  const int col0 = half * ncol;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16) + col0;
  const float max_nrm = S->max_nrm, max_kap = S->max_kap;

  int it = 0;
  int tma_pending = -1;
  for (int t = t_begin; t < t_end; ++t, ++it) {
    const uint32_t par = it & 1;
    if (tid == 0) {
      tma_pending = static_cast<int>(par);
      S->namb = 0;
      mbar_arrive_expect_tx(smem_u32(&S->tma_bar), kTileRows * d * 2);
      for (int s = 0; s < d / 64; ++s)
        tma_load_2d(&xmap, xs_u32 + s * kTileRows * 128, smem_u32(&S->tma_bar), s * 64,
                    static_cast<int>(xrow0 + static_cast<size_t>(t) * kTileRows));
      if (mbar_wait(smem_u32(&S->tma_bar), par, abort)) {
        tma_pending = -1;
        tc_fence_after();
        for (int kk = 0; kk < d / 16; ++kk) {
          int sub = kk >> 2, off = (kk & 3) * 32;
          uint64_t ad = sw128_desc(xs_u32 + sub * kTileRows * 128 + off, 16, 1024);
          uint64_t bd = sw128_desc(nus_u32 + sub * Cpad * 128 + off, 16, 1024);
          umma_f16(tmem, ad, bd, idesc, kk > 0);
        }
        umma_commit(smem_u32(&S->mma_bar));
      }
    }
    if (tid < Cpad) S->lstart[tid] = 0;
    // a CTA-uniform verdict keeps every barrier below matched
    if (__syncthreads_or(mbar_wait(smem_u32(&S->mma_bar), par, abort) ? 0 : 1)) break;
    tc_fence_after();
    const int tok = t * kTileRows + r;
    const bool valid = tok < nv;
    // ---- partial |x|^2 over this half of the dimensions; pass 1: the half's minimum
    {
      float acc = 0.f;
      const int dh = d / 2;
      for (int c = half * dh; c < (half + 1) * dh; c += 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(xs + sw128_offset(r, c, kTileRows));
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float lo = __uint_as_float(w4[q] << 16), hi = __uint_as_float(w4[q] & 0xffff0000u);
          acc = fmaf(lo, lo, fmaf(hi, hi, acc));
        }
      }
      S->xn2[half][r] = acc;
      float m = INFINITY;
      for (int q = 0; q < ncol / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(lane_addr + q * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kap + col0 + q * 32 + c);
          m = fminf(m, fminf(fminf(fmaf(-2.f, __uint_as_float(v[c]), k4.x), fmaf(-2.f, __uint_as_float(v[c + 1]), k4.y)),
                             fminf(fmaf(-2.f, __uint_as_float(v[c + 2]), k4.z), fmaf(-2.f, __uint_as_float(v[c + 3]), k4.w))));
        }
      }
      S->mh[half][r] = m;
    }
    __syncthreads();
    // ---- pass 2: every column within 2E of the row minimum is a candidate.
    // |score error| <= 2 (2^-9 + d 2^-23) |x| |nu_j| (bf16 nu, fp32 accumulation)
    // plus fp32 rounding of kappa and of the score; 2^-6 |x| max|nu| (+ a
    // relative slack) covers it with margin. Both halves compute the same thr.
    {
      const float m = fminf(S->mh[0][r], S->mh[1][r]);
      const float xn = sqrtf(S->xn2[0][r] + S->xn2[1][r]);
      const float E = ldexpf(xn * max_nrm, -6) + ldexpf(max_kap + 2.f * xn * max_nrm, -20);
      const float thr = m + 2.f * E;
      int k = 0;
      for (int q = 0; q < ncol / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(lane_addr + q * 32, v);
        tmem_wait_ld();
        uint32_t bits = 0;  // candidates of this 32-column chunk (padding has kappa = +inf)
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kap + col0 + q * 32 + c);
          bits |= (fmaf(-2.f, __uint_as_float(v[c]), k4.x) <= thr ? 1u : 0u) << c;
          bits |= (fmaf(-2.f, __uint_as_float(v[c + 1]), k4.y) <= thr ? 1u : 0u) << (c + 1);
          bits |= (fmaf(-2.f, __uint_as_float(v[c + 2]), k4.z) <= thr ? 1u : 0u) << (c + 2);
          bits |= (fmaf(-2.f, __uint_as_float(v[c + 3]), k4.w) <= thr ? 1u : 0u) << (c + 3);
        }
        while (bits) {
          const int c = __ffs(bits) - 1;
          bits &= bits - 1;
          if (k < kSlots) S->slot[r][half][k] = static_cast<int16_t>(col0 + q * 32 + c);
          ++k;
        }
      }
      S->kc[half][r] = k;
    }
    tc_fence_before();
    __syncthreads();
    // ---- rows with one candidate take it; the others are queued for fp64 re-scoring
    if (half == 0) {
      const int k0 = S->kc[0][r], k1 = S->kc[1][r];
      int L = -1;
      if (valid) {
        if (k0 + k1 == 1) {
          L = k0 ? S->slot[r][0][0] : S->slot[r][1][0];
        } else {
          S->amb[atomicAdd(&S->namb, 1)] = static_cast<int16_t>(r);
        }
      }
      S->lab[r] = L;
    }
    __syncthreads();
    // ---- one warp per ambiguous row: candidates in ascending j, strict minimum
    const int namb = S->namb;
    for (int a = warp; a < namb; a += 8) {
      const int rr = S->amb[a];
      const int k0 = S->kc[0][rr], k1 = S->kc[1][rr];
      double best = INFINITY;
      int bj = 0;
      if (k0 <= kSlots && k1 <= kSlots) {
        for (int q = 0; q < k0 + k1; ++q) {
          const int j = q < k0 ? S->slot[rr][0][q] : S->slot[rr][1][q - k0];
          const double sc = warp_score(xs, rr, nu_h + static_cast<size_t>(j) * d, kap64[j], d, lane);
          if (sc < best) {
            best = sc;
            bj = j;
          }
        }
      } else {  // too many candidates for the slots: re-score every cluster
        for (int j = 0; j < C; ++j) {
          const double sc = warp_score(xs, rr, nu_h + static_cast<size_t>(j) * d, kap64[j], d, lane);
          if (sc < best) {
            best = sc;
            bj = j;
          }
        }
      }
      if (lane == 0) S->lab[rr] = bj;
    }
    __syncthreads();
    // ---- labels out; counting sort of the tile's rows by label
    if (half == 0 && valid) {
      const int L = S->lab[r];
      assign[static_cast<size_t>(h) * nv + tok] = L;
      S->pos[r] = atomicAdd(&S->lstart[L], 1);
    }
    __syncthreads();
    if (tid < Cpad) {  // exclusive scan of the label histogram (Cpad <= 256 threads)
      const int c0 = S->lstart[tid];
      cnt[tid] += c0;
      int inc = c0;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += v;
      }
      if (lane == 31) S->wsum[warp] = inc;
      S->lstart[tid] = inc - c0;
    }
    __syncthreads();
    if (tid < Cpad) {
      int add = 0;
      for (int w = 0; w < warp; ++w) add += S->wsum[w];
      S->lstart[tid] += add;
    }
    __syncthreads();
    if (half == 0 && valid) {
      const int L = S->lab[r];
      const int p = S->lstart[L] + S->pos[r];
      S->sorted_row[p] = static_cast<int16_t>(r);
      S->sorted_lab[p] = static_cast<int16_t>(L);
    }
    __syncthreads();
    // ---- run sums in fp64: thread = (4-dimension group, slice of the sorted rows)
    {
      const int nvalid = min(kTileRows, nv - t * kTileRows);
      const int ngrp = d / 4;
      const int slices = kAssignThreads / ngrp;
      const int per = kTileRows / slices;
      const int g = tid % ngrp, sl = tid / ngrp;
      const int c4 = 4 * g;
      int cur = -1;
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      auto flush = [&]() {
        double* dst = sums + (static_cast<size_t>(h) * C + cur) * d + c4;
        atomicAdd(dst, a0);
        atomicAdd(dst + 1, a1);
        atomicAdd(dst + 2, a2);
        atomicAdd(dst + 3, a3);
      };
      const int pend = min(nvalid, (sl + 1) * per);
      for (int p = sl * per; p < pend; ++p) {
        const int L = S->sorted_lab[p];
        if (L != cur) {
          if (cur >= 0) flush();
          cur = L;
          a0 = a1 = a2 = a3 = 0.0;
        }
        const uint2 q2 = *reinterpret_cast<const uint2*>(xs + sw128_offset(S->sorted_row[p], c4, kTileRows));
        float f0 = __uint_as_float(q2.x << 16), f1 = __uint_as_float(q2.x & 0xffff0000u);
        float f2 = __uint_as_float(q2.y << 16), f3 = __uint_as_float(q2.y & 0xffff0000u);
        // components below 2^-24 count as zero (exact, order-independent sums)
        f0 = fabsf(f0) < 5.9604644775390625e-08f ? 0.f : f0;
        f1 = fabsf(f1) < 5.9604644775390625e-08f ? 0.f : f1;
        f2 = fabsf(f2) < 5.9604644775390625e-08f ? 0.f : f2;
        f3 = fabsf(f3) < 5.9604644775390625e-08f ? 0.f : f3;
        a0 += static_cast<double>(f0);
        a1 += static_cast<double>(f1);
        a2 += static_cast<double>(f2);
        a3 += static_cast<double>(f3);
      }
      if (cur >= 0) flush();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  __syncthreads();
  for (int j = tid; j < C; j += blockDim.x)
    if (cnt[j]) atomicAdd(&counts[h * C + j], cnt[j]);
  if (*abort && tid == 0) {
    report_error(err, kErrTimeoutCluster);
    if (tma_pending >= 0) {
      int dummy = 0;
      mbar_wait(smem_u32(&S->tma_bar), static_cast<uint32_t>(tma_pending), &dummy);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, tmem_cols);
}

// ---------------------------------------------------------------- finalize

// grid (C, BH), block d.
__global__ void finalize_kernel(double* __restrict__ sums, int32_t* __restrict__ counts,
                                float* __restrict__ cent, int32_t* __restrict__ sizes, int C,
                                int d) {
  const int h = blockIdx.y, j = blockIdx.x, i = threadIdx.x;
  const int n = counts[h * C + j];
  const size_t o = (static_cast<size_t>(h) * C + j) * d + i;
  if (n > 0) cent[o] = static_cast<float>(sums[o] / static_cast<double>(n));
  sums[o] = 0.0;
  __syncthreads();
  if (i == 0) {
    sizes[h * C + j] = n;
    counts[h * C + j] = 0;
  }
}

// ---------------------------------------------------------------- host side

namespace {

struct StepWs {
  double* M;
  double* nu64;
  uint16_t* nu_bf16;
  double* kappa64;
  float* kappa;
  float* nunorm;
  double* sums;
  int32_t* counts;
};

size_t carve_step(void* ws, int BH, int d, int Cmax, StepWs* out) {
  Carver cv(ws);
  int Cpad = pad64(Cmax);
  StepWs w;
  w.M = cv.take<double>(static_cast<size_t>(BH) * d * d);
  w.nu64 = cv.take<double>(static_cast<size_t>(BH) * Cmax * d);
  w.nu_bf16 = cv.take<uint16_t>(static_cast<size_t>(BH) * Cpad * d);
  w.kappa64 = cv.take<double>(static_cast<size_t>(BH) * Cpad);
  w.kappa = cv.take<float>(static_cast<size_t>(BH) * Cpad);
  w.nunorm = cv.take<float>(static_cast<size_t>(BH) * Cpad);
  w.sums = cv.take<double>(static_cast<size_t>(BH) * Cmax * d);
  w.counts = cv.take<int32_t>(static_cast<size_t>(BH) * Cmax);
  if (out) *out = w;
  return cv.used + 256;
}

int tmem_cols_for(int Cpad) {
  int c = 32;
  while (c < Cpad) c <<= 1;
  return c;
}

size_t assign_smem_bytes(int d, int Cpad) {
  return 1024 + kAssignHeader + static_cast<size_t>(kTileRows) * d * 2 +
         static_cast<size_t>(Cpad) * d * 2 + static_cast<size_t>(Cpad) * 8;
}

// One half-step. metric_cent == nullptr: identity metric.
svoo_status run_step(const svoo_shape* sh, const void* x, int C, float* cent, int32_t* sizes,
                     int32_t* assign, const float* metric_cent, const int32_t* metric_sizes,
                     int metric_C, const StepWs& w, int32_t* dev_err, cudaStream_t st,
                     int zero_C) {
  const int BH = bh_of(sh), d = sh->d, N = sh->N, nv = nvideo_of(sh);
  const int Cpad = pad64(C);
  // finalize_kernel re-zeroes what a step used, so only the first step of a
  // call clears the accumulators (for the largest cluster count of the call).
  if (zero_C > 0) {
    if (cudaMemsetAsync(w.sums, 0, sizeof(double) * BH * static_cast<size_t>(zero_C) * d, st) != cudaSuccess ||
        cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * BH * static_cast<size_t>(zero_C), st) != cudaSuccess)
      return SVOO_ERR_CUDA;
  }
  if (metric_cent) {
    const int T = d / 16;
    metric_m_kernel<<<dim3(T * (T + 1) / 2, BH), 256, 0, st>>>(metric_cent, metric_sizes, metric_C, d, w.M);
  }
  metric_nu_kernel<<<dim3(Cpad / 32, BH), 256, 0, st>>>(metric_cent ? w.M : nullptr, cent, C, Cpad, d,
                                                        w.nu64, w.nu_bf16, w.kappa64, w.kappa, w.nunorm);
  CUtensorMap xmap;
  if (encode_tiled_2d(&xmap, x, static_cast<uint64_t>(BH) * N, d, kTileRows, 64) != CUDA_SUCCESS)
    return SVOO_ERR_CUDA;
  const int ntiles = (nv + kTileRows - 1) / kTileRows;
  const int tpc = ntiles >= 128 ? 16 : (ntiles >= 16 ? 4 : 1);
  const size_t smem = assign_smem_bytes(d, Cpad);
  if (cudaFuncSetAttribute(assign_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SVOO_ERR_CUDA;
  assign_update_kernel<<<dim3((ntiles + tpc - 1) / tpc, BH), kAssignThreads, smem, st>>>(
      xmap, N, nv, d, C, Cpad, tmem_cols_for(Cpad), tpc, w.nu_bf16, w.nu64, w.kappa64, w.kappa, w.nunorm,
      assign, w.sums, w.counts, dev_err);
  finalize_kernel<<<dim3(C, BH), d, 0, st>>>(w.sums, w.counts, cent, sizes, C, d);
  return launch_status();
}

bool cluster_counts_ok(int C) { return C >= 1 && C <= 256; }

}  // namespace
}  // namespace svoo

using namespace svoo;

extern "C" size_t svoo_cluster_workspace_size(const svoo_shape* shape, int n_qc, int n_kc) {
  if (!shape_ok(shape) || !cluster_counts_ok(n_qc) || !cluster_counts_ok(n_kc)) return 0;
  return carve_step(nullptr, bh_of(shape), shape->d, n_qc > n_kc ? n_qc : n_kc, nullptr);
}

extern "C" svoo_status svoo_cluster_step(const svoo_shape* shape, const void* x, int C, float* cent,
                                         int32_t* sizes, int32_t* assign, const float* metric_cent,
                                         const int32_t* metric_sizes, int metric_C, void* workspace,
                                         size_t workspace_bytes, int32_t* dev_err, void* stream) {
  if (!shape_ok(shape) || !x || !cent || !sizes || !assign || !workspace) return SVOO_ERR_INVALID_ARG;
  if (!cluster_counts_ok(C)) return SVOO_ERR_INVALID_ARG;
  if (metric_cent && (!metric_sizes || !cluster_counts_ok(metric_C))) return SVOO_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return SVOO_ERR_INVALID_ARG;
  const int BH = bh_of(shape);
  StepWs w;
  size_t need = carve_step(workspace, BH, shape->d, C > metric_C ? C : metric_C, &w);
  if (workspace_bytes < need) return SVOO_ERR_WORKSPACE;
  return run_step(shape, x, C, cent, sizes, assign, metric_cent, metric_sizes, metric_C, w, dev_err,
                  static_cast<cudaStream_t>(stream), C);
}

extern "C" svoo_status svoo_cluster(const svoo_shape* shape, const void* q, const void* k, int n_qc,
                                    int n_kc, int iters, int warm, int32_t* q_assign,
                                    int32_t* k_assign, float* q_cent, float* k_cent,
                                    int32_t* q_sizes, int32_t* k_sizes, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_err, void* stream) {
  if (!shape_ok(shape) || !q || !k || !q_assign || !k_assign || !q_cent || !k_cent || !q_sizes ||
      !k_sizes || !workspace)
    return SVOO_ERR_INVALID_ARG;
  if (!cluster_counts_ok(n_qc) || !cluster_counts_ok(n_kc) || iters < 1 || (warm != 0 && warm != 1))
    return SVOO_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16)) return SVOO_ERR_INVALID_ARG;
  const int BH = bh_of(shape), d = shape->d, N = shape->N, nv = nvideo_of(shape);
  StepWs w;
  size_t need = carve_step(workspace, BH, d, n_qc > n_kc ? n_qc : n_kc, &w);
  if (workspace_bytes < need) return SVOO_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!warm) {
    init_centroids_kernel<<<dim3(n_qc, BH), d, 0, st>>>(static_cast<const uint16_t*>(q), N, nv, d, n_qc, q_cent);
    init_centroids_kernel<<<dim3(n_kc, BH), d, 0, st>>>(static_cast<const uint16_t*>(k), N, nv, d, n_kc, k_cent);
  }
  const int Cmax = n_qc > n_kc ? n_qc : n_kc;
  for (int it = 0; it < iters; ++it) {
    const bool ident = (it == 0 && !warm);
    svoo_status s = run_step(shape, q, n_qc, q_cent, q_sizes, q_assign, ident ? nullptr : k_cent,
                             k_sizes, n_kc, w, dev_err, st, it == 0 ? Cmax : 0);
    if (s != SVOO_OK) return s;
    s = run_step(shape, k, n_kc, k_cent, k_sizes, k_assign, q_cent, q_sizes, n_qc, w, dev_err, st, 0);
    if (s != SVOO_OK) return s;
  }
  return SVOO_OK;
}

// ---------------------------------------------------------------- allocation-free variant
//
// svoo_cluster_step_static: the same half-step as svoo_cluster_step, with its
// scratch in a fixed device array compiled into this library instead of a
// caller-provided workspace. It is for callers that may not allocate device
// memory themselves: code running inside a host framework that owns every
// device allocation through its own pool and budget, or a latency-critical
// loop whose policy forbids any allocation after start-up. The caller still
// passes the inputs and outputs.
//
// The array costs kStaticScratchBytes on every GPU that loads this library,
// until the process exits. Its device address is looked up once per device on
// the first call made with that device current (so make the first call on each
// device before any stream capture begins). Every call reuses the same array:
// each call clears the accumulators it needs before using them, and calls whose
// work overlaps on the GPU (for example on two streams) race on it.
#include <mutex>

namespace svoo {

constexpr size_t kStaticScratchBytes = static_cast<size_t>(16) << 20;
static __device__ __align__(256) unsigned char g_step_scratch[kStaticScratchBytes];

namespace {
constexpr int kMaxDevices = 128;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_step_scratch for the current device (host code must not
// use the symbol itself as a pointer: on the host it is only a stand-in).
void* scratch_address(int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  *dev_out = dev;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_step_scratch) != cudaSuccess || p == nullptr) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}
}  // namespace
}  // namespace svoo

extern "C" svoo_status svoo_cluster_step_static(const svoo_shape* shape, const void* x, int C,
                                                float* cent, int32_t* sizes, int32_t* assign,
                                                const float* metric_cent,
                                                const int32_t* metric_sizes, int metric_C,
                                                int32_t* dev_err, void* stream) {
  if (!shape_ok(shape) || !x || !cent || !sizes || !assign) return SVOO_ERR_INVALID_ARG;
  if (!cluster_counts_ok(C)) return SVOO_ERR_INVALID_ARG;
  if (metric_cent && (!metric_sizes || !cluster_counts_ok(metric_C))) return SVOO_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return SVOO_ERR_INVALID_ARG;
  const int BH = bh_of(shape);
  const int Cmax = C > metric_C ? C : metric_C;
  if (carve_step(nullptr, BH, shape->d, Cmax, nullptr) > kStaticScratchBytes)
    return SVOO_ERR_WORKSPACE;  // shape needs more than the fixed scratch holds
  int dev = 0;
  void* base = scratch_address(&dev);
  if (!base) return SVOO_ERR_CUDA;
  StepWs w;
  carve_step(base, BH, shape->d, Cmax, &w);
  return run_step(shape, x, C, cent, sizes, assign, metric_cent, metric_sizes, metric_C, w, dev_err,
                  static_cast<cudaStream_t>(stream), C);
}
