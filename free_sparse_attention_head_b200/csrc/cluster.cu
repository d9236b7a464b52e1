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

constexpr int kAssignThreads = 128;  // one token row (= TMEM lane) per thread
constexpr int kTileRows = 128;
constexpr int kMaxCandidates = 8;

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

// M[h] = sum_b n_b c_b c_b^T / sum_b n_b in fp64. grid (d/8, BH), block d
// threads; thread j owns column j of rows i0..i0+7.
__global__ void metric_m_kernel(const float* __restrict__ cent, const int32_t* __restrict__ sizes,
                                int C, int d, double* __restrict__ M) {
  extern __shared__ double sm_m[];  // [32][d] centroid chunk, then [32] sizes
  double* cch = sm_m;
  double* nch = sm_m + 32 * d;
  const int h = blockIdx.y, i0 = blockIdx.x * 8, j = threadIdx.x;
  double acc[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) acc[r] = 0.0;
  long long total = 0;
  for (int b0 = 0; b0 < C; b0 += 32) {
    int nb = min(32, C - b0);
    __syncthreads();
    for (int e = threadIdx.x; e < nb * d; e += blockDim.x)
      cch[e] = static_cast<double>(cent[(static_cast<size_t>(h) * C + b0) * d + e]);
    if (threadIdx.x < nb) nch[threadIdx.x] = static_cast<double>(sizes[h * C + b0 + threadIdx.x]);
    __syncthreads();
    for (int bb = 0; bb < nb; ++bb) {
      double n = nch[bb];
      total += static_cast<long long>(n);
      if (n == 0.0) continue;
      double cj = n * cch[bb * d + j];
#pragma unroll
      for (int r = 0; r < 8; ++r) acc[r] = fma(cch[bb * d + i0 + r], cj, acc[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    double v = total > 0 ? acc[r] / static_cast<double>(total) : (i0 + r == j ? 1.0 : 0.0);
    M[(static_cast<size_t>(h) * d + i0 + r) * d + j] = v;
  }
}

// nu_j = M mu_j (M symmetric, read by columns), kappa_j = mu_j . nu_j in fp64;
// also bf16(nu_j) for the scoring MMA, fp32 kappa and |nu_j| for its error
// bound. Clusters j in [C, Cpad) are padding (nu = 0, kappa = +inf).
// grid (Cpad/8, BH), block d threads; M == nullptr means identity.
__global__ void metric_nu_kernel(const double* __restrict__ M, const float* __restrict__ cent, int C,
                                 int Cpad, int d, double* __restrict__ nu64,
                                 uint16_t* __restrict__ nu_bf16, double* __restrict__ kappa64,
                                 float* __restrict__ kappa32, float* __restrict__ nunorm) {
  extern __shared__ double sm_nu[];  // [8][d] mu rows, [8][4][2] reduction scratch
  double* mu = sm_nu;
  double* red = sm_nu + 8 * d;
  const int h = blockIdx.y, j0 = blockIdx.x * 8, i = threadIdx.x;
  for (int e = threadIdx.x; e < 8 * d; e += blockDim.x) {
    int r = e / d, c = e % d;
    mu[e] = (j0 + r < C) ? static_cast<double>(cent[(static_cast<size_t>(h) * C + j0 + r) * d + c]) : 0.0;
  }
  __syncthreads();
  double acc[8];
  if (M) {
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = 0.0;
    const double* Mh = M + static_cast<size_t>(h) * d * d;
    for (int l = 0; l < d; ++l) {
      double m = Mh[static_cast<size_t>(l) * d + i];
#pragma unroll
      for (int r = 0; r < 8; ++r) acc[r] = fma(m, mu[r * d + l], acc[r]);
    }
  } else {
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = mu[r * d + i];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    int j = j0 + r;
    size_t o = (static_cast<size_t>(h) * Cpad + j) * d + i;
    if (j < C) nu64[(static_cast<size_t>(h) * C + j) * d + i] = acc[r];
    __nv_bfloat16 b = __float2bfloat16_rn(j < C ? static_cast<float>(acc[r]) : 0.f);
    nu_bf16[o] = *reinterpret_cast<uint16_t*>(&b);
    double k1 = mu[r * d + i] * acc[r];
    double k2 = acc[r] * acc[r];
    for (int s = 16; s > 0; s >>= 1) {
      k1 += __shfl_xor_sync(0xffffffffu, k1, s);
      k2 += __shfl_xor_sync(0xffffffffu, k2, s);
    }
    if (lane == 0) {
      red[(r * 4 + warp) * 2 + 0] = k1;
      red[(r * 4 + warp) * 2 + 1] = k2;
    }
  }
  __syncthreads();
  if (threadIdx.x < 8) {
    int r = threadIdx.x, j = j0 + r;
    double k1 = 0.0, k2 = 0.0;
    for (int w = 0; w < nwarp; ++w) {
      k1 += red[(r * 4 + w) * 2 + 0];
      k2 += red[(r * 4 + w) * 2 + 1];
    }
    kappa64[h * Cpad + j] = j < C ? k1 : INFINITY;
    kappa32[h * Cpad + j] = j < C ? static_cast<float>(k1) : INFINITY;
    nunorm[h * Cpad + j] = j < C ? static_cast<float>(sqrt(k2)) : 0.f;
  }
}

// ---------------------------------------------------------------- assign + update

struct AssignSmem {
  int abort;
  uint32_t tmem_base;
  uint64_t tma_bar;
  uint64_t mma_bar;
  int lab[kTileRows];
  uint32_t keys[kTileRows];
};

constexpr int kAssignHeader = 2048;  // AssignSmem, padded so the X tile stays 1024-aligned
static_assert(sizeof(AssignSmem) <= kAssignHeader, "header overflow");

// grid (ceil(ntiles / tiles_per_cta), BH), block 128.
// Dynamic smem: [AssignSmem, 2 KB][X tile 128 x d bf16][nu Cpad x d bf16][kappa][nunorm]
__global__ void __launch_bounds__(kAssignThreads)
    assign_update_kernel(const __grid_constant__ CUtensorMap xmap, int N, int nv, int d, int C,
                         int Cpad, int tmem_cols, int tiles_per_cta,
                         const uint16_t* __restrict__ nu_bf16, const double* __restrict__ nu64,
                         const double* __restrict__ kappa64, const float* __restrict__ kappa_g,
                         const float* __restrict__ nunorm_g,
                         int32_t* __restrict__ assign, double* __restrict__ sums,
                         int32_t* __restrict__ counts, int* __restrict__ err) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AssignSmem* S = reinterpret_cast<AssignSmem*>(base);
  uint8_t* xs = base + kAssignHeader;
  uint8_t* nus = xs + kTileRows * d * 2;
  float* kap = reinterpret_cast<float*>(nus + static_cast<size_t>(Cpad) * d * 2);
  float* nrm = kap + Cpad;

  const int h = blockIdx.y, tid = threadIdx.x, warp = tid >> 5;
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
  // nu (bf16) into the 128B-swizzled K-major layout the MMA expects.
  {
    const int chunks = d / 8;
    const uint4* src = reinterpret_cast<const uint4*>(nu_bf16 + static_cast<size_t>(h) * Cpad * d);
    for (int e = tid; e < Cpad * chunks; e += blockDim.x) {
      int j = e / chunks, c = e % chunks;
      *reinterpret_cast<uint4*>(nus + sw128_offset(j, c * 8, Cpad)) = src[e];
    }
    for (int j = tid; j < Cpad; j += blockDim.x) {
      kap[j] = kappa_g[h * Cpad + j];
      nrm[j] = nunorm_g[h * Cpad + j];
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

  int it = 0;
  int tma_pending = -1;  // parity of a TMA phase issued but not yet seen complete
  for (int t = t_begin; t < t_end; ++t, ++it) {
    const uint32_t par = it & 1;
    if (tid == 0) {
      tma_pending = static_cast<int>(par);
      mbar_arrive_expect_tx(smem_u32(&S->tma_bar), kTileRows * d * 2);
      for (int s = 0; s < d / 64; ++s)
        tma_load_2d(&xmap, xs_u32 + s * kTileRows * 128, smem_u32(&S->tma_bar), s * 64,
                    static_cast<int>(xrow0 + static_cast<size_t>(t) * kTileRows));
      bool ok = mbar_wait(smem_u32(&S->tma_bar), par, abort);
      if (ok) {
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
    // warp-uniform verdict: the tcgen05.ld below is warp-collective
    if (!__all_sync(0xffffffffu, mbar_wait(smem_u32(&S->mma_bar), par, abort))) break;
    tc_fence_after();

    // ---- per-token argmin with error bound and fp32 recheck
    const int r = tid;
    const int tok = t * kTileRows + r;
    const bool valid = tok < nv;
    const uint8_t* xrow = xs;  // element (r, c) at sw128_offset(r, c, 128)
    float xn2 = 0.f;
    for (int c = 0; c < d; ++c) {
      float v = bf16_to_f32(*reinterpret_cast<const uint16_t*>(xrow + sw128_offset(r, c, kTileRows)));
      xn2 = fmaf(v, v, xn2);
    }
    // |x.nu - acc| <= 2^-8 |x||nu| covers bf16 rounding of nu (2^-9) plus the
    // fp32 accumulation; the score kappa - 2 x.nu therefore errs by at most
    // 2^-7 |x||nu|. Use 2^-6 for margin.
    const float eps_x = ldexpf(sqrtf(xn2), -6);
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float U = INFINITY;
    for (int q = 0; q < Cpad / 32; ++q) {
      uint32_t v[32];
      tmem_ld32(lane_addr + q * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        int j = q * 32 + c;
        float s = kap[j] - 2.f * __uint_as_float(v[c]);
        U = fminf(U, s + eps_x * nrm[j]);
      }
    }
    int cand[kMaxCandidates];
    int ncand = 0;
    bool overflow = false;
    for (int q = 0; q < Cpad / 32; ++q) {
      uint32_t v[32];
      tmem_ld32(lane_addr + q * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        int j = q * 32 + c;
        float s = kap[j] - 2.f * __uint_as_float(v[c]);
        if (s - eps_x * nrm[j] <= U) {
          if (ncand < kMaxCandidates) cand[ncand] = j;
          else overflow = true;
          ++ncand;
        }
      }
    }
    tc_fence_before();
    // Decision: a single candidate is the argmin; otherwise the candidates
    // are re-scored exactly as the definition reads, kappa_j - 2 x.nu_j in
    // fp64 (nu, kappa from the fp64 metric), ties to the smaller j.
    int best_j = 0;
    auto exact_score = [&](int j) -> double {
      const double* nj = nu_h + static_cast<size_t>(j) * d;
      double dot = 0.0;
      for (int c = 0; c < d; ++c) {
        float xv = bf16_to_f32(*reinterpret_cast<const uint16_t*>(xrow + sw128_offset(r, c, kTileRows)));
        dot = fma(static_cast<double>(xv), __ldg(nj + c), dot);
      }
      return kap64[j] - 2.0 * dot;
    };
    if (valid) {
      if (ncand == 1) {
        best_j = cand[0];
      } else {
        double best = INFINITY;
        const int n_eval = overflow ? C : ncand;
        for (int k = 0; k < n_eval; ++k) {
          const int j = overflow ? k : cand[k < kMaxCandidates ? k : 0];
          const double s = exact_score(j);
          if (s < best) {  // candidates ascend in j: ties keep the smaller j
            best = s;
            best_j = j;
          }
        }
      }
      assign[static_cast<size_t>(h) * nv + tok] = best_j;
    }
    S->lab[r] = valid ? best_j : -1;
    S->keys[r] = (static_cast<uint32_t>(valid ? best_j + 1 : 0) << 8) | static_cast<uint32_t>(r);
    __syncthreads();

    // ---- bitonic sort of (label, row) keys, 128 entries, one per thread
    for (int k = 2; k <= kTileRows; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        int ixj = r ^ jj;
        if (ixj > r) {
          uint32_t a = S->keys[r], b = S->keys[ixj];
          bool up = (r & k) == 0;
          if ((a > b) == up) {
            S->keys[r] = b;
            S->keys[ixj] = a;
          }
        }
        __syncthreads();
      }
    }
    // ---- run sums (exact fp64) -> atomics; thread = dimension
    if (r < d) {
      int cur = -1;
      double acc = 0.0;
      for (int p = 0; p < kTileRows; ++p) {
        uint32_t key = S->keys[p];
        int lbl = static_cast<int>(key >> 8) - 1;
        if (lbl < 0) continue;
        int row = key & 255;
        if (lbl != cur) {
          if (cur >= 0) atomicAdd(&sums[(static_cast<size_t>(h) * C + cur) * d + r], acc);
          cur = lbl;
          acc = 0.0;
        }
        float v = bf16_to_f32(*reinterpret_cast<const uint16_t*>(xrow + sw128_offset(row, r, kTileRows)));
        if (fabsf(v) < 5.9604644775390625e-08f) v = 0.f;  // 2^-24
        acc += static_cast<double>(v);
      }
      if (cur >= 0) atomicAdd(&sums[(static_cast<size_t>(h) * C + cur) * d + r], acc);
    }
    if (r == (d < kTileRows ? d : 0)) {
      // one thread counts the runs (d < 128: a thread outside the sum loop)
      int cur = -1, len = 0;
      for (int p = 0; p < kTileRows; ++p) {
        int lbl = static_cast<int>(S->keys[p] >> 8) - 1;
        if (lbl < 0) continue;
        if (lbl != cur) {
          if (cur >= 0) atomicAdd(&counts[h * C + cur], len);
          cur = lbl;
          len = 0;
        }
        ++len;
      }
      if (cur >= 0) atomicAdd(&counts[h * C + cur], len);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  if (*abort && tid == 0) {
    report_error(err, kErrTimeoutCluster);
    // never leave with a copy still writing into this CTA's shared memory
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
  int Cpad = pad32(Cmax);
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
  const int Cpad = pad32(C);
  // finalize_kernel re-zeroes what a step used, so only the first step of a
  // call clears the accumulators (for the largest cluster count of the call).
  if (zero_C > 0) {
    if (cudaMemsetAsync(w.sums, 0, sizeof(double) * BH * static_cast<size_t>(zero_C) * d, st) != cudaSuccess ||
        cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * BH * static_cast<size_t>(zero_C), st) != cudaSuccess)
      return SVOO_ERR_CUDA;
  }
  if (metric_cent) {
    metric_m_kernel<<<dim3(d / 8, BH), d, (32 * d + 32) * sizeof(double), st>>>(metric_cent, metric_sizes,
                                                                                metric_C, d, w.M);
  }
  metric_nu_kernel<<<dim3(Cpad / 8, BH), d, (8 * d + 64) * sizeof(double), st>>>(
      metric_cent ? w.M : nullptr, cent, C, Cpad, d, w.nu64, w.nu_bf16, w.kappa64, w.kappa, w.nunorm);
  CUtensorMap xmap;
  if (encode_tiled_2d(&xmap, x, static_cast<uint64_t>(BH) * N, d, kTileRows, 64) != CUDA_SUCCESS)
    return SVOO_ERR_CUDA;
  const int ntiles = (nv + kTileRows - 1) / kTileRows;
  const int tpc = ntiles >= 64 ? 8 : 1;
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
