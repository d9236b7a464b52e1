// cluster.cu -- per-head bidirectional QK co-clustering (SVOO abstract; iCATS
// sections 3.1 and 4.1): k-means of the query tokens and of the key tokens,
// each side's distance being the interaction error under the metric of the
// other side's clusters, M = sum_b n_b c_b c_b^T / sum_b n_b (identity in the
// cold first query step).
//
// Kernels of one half-step (one side):
//   metric_m_kernel   M from the other side's centroids and sizes (fp64)
//   metric_nu_kernel  nu_j = M mu_j, kappa_j = mu_j . nu_j (fp64), |nu_j|, and
//                     nu_j split into two bf16 rows (hi + lo)
//   assign_kernel     persistent, warp-specialised: tcgen05 MMAs of 128-token
//                     tiles against [nu_hi | nu_lo] into double-buffered TMEM;
//                     per token the score kappa_j - 2 x.nu_j is bounded by the
//                     MMA error, a token with a single candidate takes it and
//                     the rest are re-scored in fp64 (ties to the smaller j);
//                     member sums in fp64 (exact, so order-independent) and
//                     counts, added atomically.
//   finalize_kernel   centroid = fp32(sum / count), empty clusters keep
//                     theirs; resets the sums for the next half-step.
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
// T = d/64 output blocks of 64 x 64 per side (upper triangle only; an
// off-diagonal block is written to both (i, j) and (j, i), so M is exactly
// symmetric), block 512 = two groups of 16 x 16 threads that take alternate
// 32-cluster chunks (their partial blocks are added at the end, group 0's
// plus group 1's); thread (ty, tx) of a group owns rows i0 + 4ty .. +3 and
// columns j0 + {2tx, 2tx+1, 32+2tx, 33+2tx}. The next chunk's values are
// fetched into registers while the current one is used.
constexpr int kMBlk = 64;
constexpr int kMChunk = 32;
constexpr int kMThreads = 512;

__global__ void __launch_bounds__(kMThreads)
    metric_m_kernel(const float* __restrict__ cent, const int32_t* __restrict__ sizes, int C, int d,
                    double* __restrict__ M) {
  extern __shared__ __align__(16) double msm[];   // per group: as[32][64], bs[32][64]
  __shared__ long long total_s;
  const int h = blockIdx.y, T = d / kMBlk;
  int t = blockIdx.x, bi = 0;
  while (t >= T - bi) {  // upper-triangle block index -> (bi, bj), bi <= bj
    t -= T - bi;
    ++bi;
  }
  const int bj = bi + t;
  const int i0 = bi * kMBlk, j0 = bj * kMBlk;
  const int grp = threadIdx.x >> 8, gt = threadIdx.x & 255;
  const int ty = gt >> 4, tx = gt & 15;
  double* as = msm + grp * 2 * kMChunk * kMBlk;
  double* bs = as + kMChunk * kMBlk;
  const float* ch = cent + static_cast<size_t>(h) * C * d;
  const int32_t* sh = sizes + static_cast<size_t>(h) * C;
  constexpr int kPer = kMChunk * kMBlk / 256;  // 8 staged elements per thread
  float fa[kPer], fb[kPer];
  int nb_[kPer];
  auto fetch = [&](int b0) {
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int e = gt + 256 * q;
      const int bb = e / kMBlk, c = e % kMBlk;
      fa[q] = 0.f;
      fb[q] = 0.f;
      nb_[q] = 0;
      if (b0 + bb < C) {
        const float* cb = ch + static_cast<size_t>(b0 + bb) * d;
        fa[q] = cb[i0 + c];
        fb[q] = cb[j0 + c];
        nb_[q] = sh[b0 + bb];
      }
    }
  };
  double acc[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.0;
  const int nchunks = (C + kMChunk - 1) / kMChunk;
  const int rounds = (nchunks + 1) / 2;  // both groups run the same number of rounds
  fetch(grp * kMChunk);
  for (int rd = 0; rd < rounds; ++rd) {
    const int b0 = (2 * rd + grp) * kMChunk;
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int e = gt + 256 * q;
      as[e] = static_cast<double>(nb_[q]) * static_cast<double>(fa[q]);
      bs[e] = static_cast<double>(fb[q]);
    }
    __syncthreads();
    if (b0 + 2 * kMChunk < C) fetch(b0 + 2 * kMChunk);
    const int nb = max(0, min(kMChunk, C - b0));
    for (int bb = 0; bb < nb; ++bb) {
      const double2 a01 = *reinterpret_cast<const double2*>(&as[bb * kMBlk + 4 * ty]);
      const double2 a23 = *reinterpret_cast<const double2*>(&as[bb * kMBlk + 4 * ty + 2]);
      const double2 b01 = *reinterpret_cast<const double2*>(&bs[bb * kMBlk + 2 * tx]);
      const double2 b23 = *reinterpret_cast<const double2*>(&bs[bb * kMBlk + 32 + 2 * tx]);
      const double av[4] = {a01.x, a01.y, a23.x, a23.y};
      const double bv[4] = {b01.x, b01.y, b23.x, b23.y};
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fma(av[u], bv[v], acc[u][v]);
    }
  }
  if (threadIdx.x < 32) {
    long long s = 0;
    for (int b = threadIdx.x; b < C; b += 32) s += sh[b];
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) total_s = s;
  }
  // group 1's partial block joins group 0's through shared memory
  __syncthreads();
  double* part = msm;  // [16 ty][16 tx][16]
  if (grp == 1) {
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) part[gt * 16 + u * 4 + v] = acc[u][v];
  }
  __syncthreads();
  if (grp == 1) return;
  const long long total = total_s;
  double* Mh = M + static_cast<size_t>(h) * d * d;
  const int jc[4] = {2 * tx, 2 * tx + 1, 32 + 2 * tx, 33 + 2 * tx};
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int i = i0 + 4 * ty + u, j = j0 + jc[v];
      const double sum = acc[u][v] + part[gt * 16 + u * 4 + v];
      const double val = total > 0 ? sum / static_cast<double>(total) : (i == j ? 1.0 : 0.0);
      Mh[static_cast<size_t>(i) * d + j] = val;
      if (bi != bj) Mh[static_cast<size_t>(j) * d + i] = val;
    }
}
constexpr size_t kMetricMSmem = 2 * 2 * kMChunk * kMBlk * sizeof(double);  // 64 KB

// nu_j = M mu_j and kappa_j = mu_j . nu_j in fp64; nu_j also as the pair of
// bf16 rows nu_hi = bf16(nu_j), nu_lo = bf16(nu_j - nu_hi) that the scoring
// MMA consumes (their sum is nu_j to 2^-18 relative), and |nu_j|. Clusters j
// in [C, CP) are padding (nu = 0, kappa = +inf). grid (CP/32, BH), block 128:
// warp w owns clusters j0 + 8w .. +7, lane owns dimensions 2 lane, 2 lane + 1
// (and 64 + the same for d = 128). Rows of M arrive 16 at a time by cp.async,
// one chunk ahead. M == nullptr means the identity.
constexpr int kNuRows = 16;
constexpr int kNuMuStride = 130;  // doubles per staged centroid row (keeps 16-byte alignment)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(128)
    metric_nu_kernel(const double* __restrict__ M, const float* __restrict__ cent, int C, int CP,
                     int d, double* __restrict__ nu64, uint16_t* __restrict__ nu_hi,
                     uint16_t* __restrict__ nu_lo, double* __restrict__ kappa64,
                     float* __restrict__ kappa32, float* __restrict__ nunorm) {
  extern __shared__ __align__(16) double nsm[];
  double* mu = nsm;                          // [32][kNuMuStride]
  double* mch = mu + 32 * kNuMuStride;       // two buffers of [16][d]
  const int h = blockIdx.y, j0 = blockIdx.x * 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double* Mh = M ? M + static_cast<size_t>(h) * d * d : nullptr;
  auto stage = [&](int chunk) {  // rows 16 chunk .. +15 of M into buffer chunk % 2
    double* dst = mch + (chunk & 1) * kNuRows * d;
    const double* src = Mh + static_cast<size_t>(chunk) * kNuRows * d;
    for (int e = threadIdx.x; e < kNuRows * d / 2; e += blockDim.x) cp_async16(dst + 2 * e, src + 2 * e);
    cp_async_commit();
  };
  if (Mh) stage(0);
  for (int e = threadIdx.x; e < 32 * d; e += blockDim.x) {
    const int r = e / d, c = e % d;
    mu[r * kNuMuStride + c] = (j0 + r < C) ? static_cast<double>(cent[(static_cast<size_t>(h) * C + j0 + r) * d + c]) : 0.0;
  }
  const int nd = d == 128 ? 4 : 2;  // dimensions per lane
  const int dim[4] = {2 * lane, 2 * lane + 1, 64 + 2 * lane, 65 + 2 * lane};
  const double* mw = mu + 8 * warp * kNuMuStride;
  double acc[8][4];  // [cluster][dimension]
#pragma unroll
  for (int u = 0; u < 8; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) acc[u][v] = 0.0;
  if (Mh) {
    const int nchunks = d / kNuRows;
    for (int ck = 0; ck < nchunks; ++ck) {
      if (ck + 1 < nchunks) {
        stage(ck + 1);
        cp_async_wait<1>();
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();
      const double* mb = mch + (ck & 1) * kNuRows * d;
#pragma unroll 4
      for (int l = 0; l < kNuRows; ++l) {
        // M symmetric: nu_j[i] = sum_l M[l][i] mu_j[l]
        const double2 m01 = *reinterpret_cast<const double2*>(&mb[l * d + 2 * lane]);
        double2 m23 = make_double2(0.0, 0.0);
        if (d == 128) m23 = *reinterpret_cast<const double2*>(&mb[l * d + 64 + 2 * lane]);
        const double mv[4] = {m01.x, m01.y, m23.x, m23.y};
        const int li = ck * kNuRows + l;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const double m_u = mw[u * kNuMuStride + li];
#pragma unroll
          for (int v = 0; v < 4; ++v) acc[u][v] = fma(mv[v], m_u, acc[u][v]);
        }
      }
      __syncthreads();  // this buffer is refilled two chunks later
    }
  } else {
    __syncthreads();
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = v < nd ? mw[u * kNuMuStride + dim[v]] : 0.0;
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int j = j0 + 8 * warp + u;
    double k1 = 0.0, k2 = 0.0;
    uint16_t hb[4], lb[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const double a = (j < C && v < nd) ? acc[u][v] : 0.0;
      if (v < nd) {
        k1 = fma(mw[u * kNuMuStride + dim[v]], a, k1);
        k2 = fma(a, a, k2);
      }
      const __nv_bfloat16 bh = __float2bfloat16_rn(static_cast<float>(a));
      const double rest = a - static_cast<double>(__bfloat162float(bh));
      const __nv_bfloat16 bl = __float2bfloat16_rn(static_cast<float>(rest));
      hb[v] = *reinterpret_cast<const uint16_t*>(&bh);
      lb[v] = *reinterpret_cast<const uint16_t*>(&bl);
    }
    const size_t row = static_cast<size_t>(h) * CP + j;
    uint32_t* oh = reinterpret_cast<uint32_t*>(nu_hi + row * d);
    uint32_t* ol = reinterpret_cast<uint32_t*>(nu_lo + row * d);
    oh[lane] = hb[0] | (static_cast<uint32_t>(hb[1]) << 16);
    ol[lane] = lb[0] | (static_cast<uint32_t>(lb[1]) << 16);
    if (d == 128) {
      oh[32 + lane] = hb[2] | (static_cast<uint32_t>(hb[3]) << 16);
      ol[32 + lane] = lb[2] | (static_cast<uint32_t>(lb[3]) << 16);
    }
    if (j < C) {
      double* on = nu64 + (static_cast<size_t>(h) * C + j) * d;
      *reinterpret_cast<double2*>(on + 2 * lane) = make_double2(acc[u][0], acc[u][1]);
      if (d == 128) *reinterpret_cast<double2*>(on + 64 + 2 * lane) = make_double2(acc[u][2], acc[u][3]);
    }
    for (int o = 16; o > 0; o >>= 1) {
      k1 += __shfl_xor_sync(0xffffffffu, k1, o);
      k2 += __shfl_xor_sync(0xffffffffu, k2, o);
    }
    if (lane == 0) {
      kappa64[h * CP + j] = j < C ? k1 : INFINITY;
      kappa32[h * CP + j] = j < C ? static_cast<float>(k1) : INFINITY;
      nunorm[h * CP + j] = j < C ? static_cast<float>(sqrt(k2)) : 0.f;
    }
  }
}
inline size_t metric_nu_smem(int d) { return (32 * kNuMuStride + 2 * kNuRows * d) * sizeof(double); }

// ---------------------------------------------------------------- assign + update
//
// Persistent, warp-specialised kernel, one CTA per SM, each CTA walking a
// contiguous stretch of the (head, 128-token tile) sequence. Tile i uses X
// buffer i % 2 in shared memory and TMEM accumulator i % 2 (CP fp32 columns).
//   producer (warp 0)   TMA of the X tile, then one tcgen05 chain per tile:
//                       u = X . nu_hi^T + X . nu_lo^T + 1 . (-kappa/2)^T, the
//                       last term a 16-wide K chunk of ones against -kappa_j/2
//                       split into three bf16 parts, so u_j = x.nu_j - kappa_j/2
//                       and the score is kappa_j - 2 x.nu_j = -2 u_j.
//   scorers (warps 8-15) thread (row r, column half): |x|^2 over half of the
//                       dimensions (then the X buffer goes back), the half's
//                       maximum of u, and, with the row maximum U and the error
//                       bound E, its candidates u_j >= U - 2E (they contain the
//                       exact argmin of the score; then the accumulator goes
//                       back). A row with one candidate takes it; the others
//                       are deferred with their candidate list.
//   summers (warps 1-7) warp w owns rows [128(w-1)/7, 128w/7) of every tile:
//                       member sums of the labelled rows (re-read from L2), a
//                       run of equal labels in token order summed in fp32 and
//                       added with one vector atomic per lane, and the deferred
//                       rows, decided from the shared-memory nu copies or, inside
//                       that bound, by an fp64 re-score (ties to the smaller j).
//
// Error bound: nu_hi + nu_lo equals nu to 2^-18 relative and the three kappa
// parts give kappa to 2^-26; the MMA's fp32 accumulation of 2d + 3 exact
// products adds at most (2d + 3) 2^-23 of the sum of their magnitudes, at most
// |x||nu_j| (1 + 2^-8) + |kappa_j| / 2. E = 2^-13 (|x| max|nu| + max|kappa| / 2)
// bounds |u_computed - u| with a factor of two to spare.

constexpr int kScorerWarps = 8;
constexpr int kSummerWarps = 7;
// warp 0 is the producer; the summers take the next warp ids, the scorers the last
constexpr int kFirstSummer = 1;
constexpr int kFirstScorer = kFirstSummer + kSummerWarps;
constexpr int kAssignWarps = 1 + kScorerWarps + kSummerWarps;
constexpr int kAssignThreads = kAssignWarps * 32;
constexpr int kScorers = kScorerWarps * 32;
constexpr int kSummers = kSummerWarps * 32;
constexpr int kTileRows = 128;
constexpr int kHalfCand = 4;             // candidates kept per column half
constexpr int kAssignHeader = 16384;     // AssignSmem, keeps the X buffers 1024-aligned
constexpr int kExtraK = 16;              // the kappa chunk of the MMA
// named barriers: 1..4 the two scorer warps of a TMEM lane quarter, 5 all scorers
constexpr int kBarScorers = 5;

struct AssignSmem {
  uint64_t x_full[2], x_free[2], t_full[2], t_free[2], l_full[2], l_free[2];
  uint32_t tmem_base;
  int abort;
  float max_nrm;
  float max_kap;
  float xq[2][kTileRows];                  // |x|^2 per column half's dimensions
  float mh[2][kTileRows];                  // per-half maxima of u
  uint8_t kc[2][kTileRows];                // candidates per half (saturating)
  int16_t cand[2][kTileRows][kHalfCand];
  // published per tile parity for the summers
  int16_t lab[2][kTileRows];               // label; -1 not a video token; -2 deferred
  uint32_t defmask[2][kTileRows / 32];     // deferred rows of the tile, one bit per row
  int8_t def_n[2][kTileRows];              // deferred row: candidates listed (0 = all)
  int16_t def_cand[2][kTileRows][2 * kHalfCand];
};
static_assert(sizeof(AssignSmem) <= kAssignHeader, "assign header overflow");

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// barrier over a group of warps that also ORs a flag across them
__device__ __forceinline__ int named_sync_or(int id, int threads, int flag) {
  int r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.b32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.b32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(flag), "r"(id), "r"(threads)
      : "memory");
  return r;
}

// Shared memory matrix descriptor without swizzle (K-major): 8-row x 16-byte
// core matrices, `lbo` bytes between the two K halves of a 16-element row
// chunk, `sbo` bytes between 8-row groups.
__device__ __forceinline__ uint64_t plain_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFF);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFF) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;  // layout type 0: no swizzle
}

// byte offset of element (row, k) of a [rows][16] bf16 tile in that layout
// (lbo = 128, sbo = 256)
__device__ __forceinline__ uint32_t plain_offset(int row, int k) {
  return static_cast<uint32_t>((row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float f) {
  const __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&b);
}

// Member sums are fp32: a run of equal labels among a warp's rows of a tile
// (at most 19 rows, token order) is summed in registers and added with one
// vector atomic per lane (lane l owns dimensions 4l .. 4l+3, or 2l, 2l+1 for
// d = 64), so a run costs the L2 one operation per 32-byte sector.
template <int D>
__device__ __forceinline__ void flush_row(float* dst, float v0, float v1, float v2, float v3, int lane) {
  if (D == 128)
    atomicAdd(reinterpret_cast<float4*>(dst) + lane, make_float4(v0, v1, v2, v3));
  else
    atomicAdd(reinterpret_cast<float2*>(dst) + lane, make_float2(v0, v1));
}

constexpr int kSumRows = (kTileRows + kSummerWarps - 1) / kSummerWarps;  // rows per summer warp

// Decides a deferred row (its candidates listed in ascending j, or all
// clusters). First, in fp32, t_j = x.(nu_hi + nu_lo)_j + (-kappa_j / 2 in three
// parts): the products are exact and 16 roundings of at most 2^-24 of the sum
// of magnitudes are added, so |t_j - u_j| <= 2^-18 |x||nu_j| + 2^-26 |kappa_j|
// + 2^-20 (|x||nu_j| + |kappa_j| / 2). If one candidate stays within twice that
// of the maximum it is the answer; otherwise the survivors are re-scored
// exactly, kappa_j - 2 x.nu_j from the fp64 nu and kappa, ties to the smaller j.
// One warp; lane owns dimensions 4 lane .. 4 lane + 3 (2 lane, 2 lane + 1 for d = 64):
// xa holds the first two of them, xb the other two.
template <int D, int CP>
__device__ __forceinline__ float approx_t(int j, float x0, float x1, float x2, float x3, const uint8_t* nuh,
                                         const uint8_t* nul, const uint8_t* kparts, int lane) {
  auto bf = [](const uint8_t* base, uint32_t off) {
    return __uint_as_float(static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(base + off)) << 16);
  };
  constexpr int kPer = D / 32;  // dimensions per lane (4 or 2), consecutive
  const uint32_t o0 = sw128_offset(j, kPer * lane, CP);
  float p = x0 * bf(nuh, o0);
  p = fmaf(x0, bf(nul, o0), p);
  p = fmaf(x1, bf(nuh, o0 + 2), p);
  p = fmaf(x1, bf(nul, o0 + 2), p);
  if (D == 128) {
    p = fmaf(x2, bf(nuh, o0 + 4), p);
    p = fmaf(x2, bf(nul, o0 + 4), p);
    p = fmaf(x3, bf(nuh, o0 + 6), p);
    p = fmaf(x3, bf(nul, o0 + 6), p);
  }
  for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
  return p + bf(kparts, plain_offset(j, 0)) + bf(kparts, plain_offset(j, 1)) + bf(kparts, plain_offset(j, 2));
}

template <int D, int CP>
__device__ __noinline__ int decide_deferred(const AssignSmem* S, int b, int rr, uint32_t xa, uint32_t xb,
                               const uint8_t* nuh, const uint8_t* nul, const uint8_t* kparts,
                               float max_nrm, float max_kap, const double* __restrict__ nu_h,
                               const double* __restrict__ kap_h, int C, int lane) {
  const float x0 = __uint_as_float(xa << 16), x1 = __uint_as_float(xa & 0xffff0000u);
  const float x2 = __uint_as_float(xb << 16), x3 = __uint_as_float(xb & 0xffff0000u);
  float xx = x0 * x0 + x1 * x1 + x2 * x2 + x3 * x3;
  for (int o = 16; o > 0; o >>= 1) xx += __shfl_xor_sync(0xffffffffu, xx, o);
  const float E2 = ldexpf(sqrtf(xx) * max_nrm + 0.5f * max_kap, -16);  // twice the bound, with margin
  const int n = S->def_n[b][rr];
  constexpr int kMax = 2 * kHalfCand;
  float t[kMax];
  float T = -INFINITY;
  if (n > 0) {  // listed candidates: all evaluated together
#pragma unroll
    for (int q = 0; q < kMax; ++q) {
      t[q] = -INFINITY;
      if (q < n) t[q] = approx_t<D, CP>(S->def_cand[b][rr][q], x0, x1, x2, x3, nuh, nul, kparts, lane);
      T = fmaxf(T, t[q]);
    }
  } else {
    for (int j = 0; j < C; ++j) T = fmaxf(T, approx_t<D, CP>(j, x0, x1, x2, x3, nuh, nul, kparts, lane));
  }
  int survivors = 0, only = 0;
  if (n > 0) {
#pragma unroll
    for (int q = 0; q < kMax; ++q)
      if (q < n && t[q] >= T - E2) {
        ++survivors;
        only = S->def_cand[b][rr][q];
      }
  } else {
    for (int j = 0; j < C; ++j)
      if (approx_t<D, CP>(j, x0, x1, x2, x3, nuh, nul, kparts, lane) >= T - E2) {
        ++survivors;
        only = j;
      }
  }
  if (survivors == 1) return only;
  // exact: the survivors in ascending j, strict minimum of kappa_j - 2 x.nu_j
  const double d0 = x0, d1 = x1, d2 = x2, d3 = x3;
  double best = INFINITY;
  int bj = 0;
  const int J = n > 0 ? n : C;
  for (int q = 0; q < J; ++q) {
    const int j = n > 0 ? static_cast<int>(S->def_cand[b][rr][q]) : q;
    if (approx_t<D, CP>(j, x0, x1, x2, x3, nuh, nul, kparts, lane) < T - E2) continue;
    const double* nj = nu_h + static_cast<size_t>(j) * D + (D / 32) * lane;
    const double2 na = *reinterpret_cast<const double2*>(nj);
    double e = fma(d0, na.x, d1 * na.y);
    if (D == 128) {
      const double2 nb = *reinterpret_cast<const double2*>(nj + 2);
      e = fma(d2, nb.x, fma(d3, nb.y, e));
    }
    for (int o = 16; o > 0; o >>= 1) e += __shfl_xor_sync(0xffffffffu, e, o);
    const double sc = kap_h[j] - 2.0 * e;
    if (sc < best) {
      best = sc;
      bj = j;
    }
  }
  return bj;
}

// grid: min(#SMs, B*H*tiles) CTAs, block kAssignThreads. Dynamic smem:
// [AssignSmem 16 KB][X 2 x 128 x D bf16][nu_hi CP x D][nu_lo CP x D][ones 128 x 16][kappa parts CP x 16]
template <int D, int CP>
__global__ void __launch_bounds__(kAssignThreads, 1)
    assign_kernel(const __grid_constant__ CUtensorMap xmap, const uint16_t* __restrict__ x, int N,
                  int nv, int C, int BH, const uint16_t* __restrict__ nu_hi,
                  const uint16_t* __restrict__ nu_lo, const double* __restrict__ nu64,
                  const double* __restrict__ kappa64, const float* __restrict__ nunorm,
                  int32_t* __restrict__ assign, float* __restrict__ sums,
                  int32_t* __restrict__ counts, int* __restrict__ err) {
  constexpr int kHalfCols = CP / 2;                 // score columns per scorer thread
  constexpr int kChunks = kHalfCols / 32;           // 32-column TMEM loads per pass
  constexpr uint32_t kXBytes = kTileRows * D * 2;
  constexpr uint32_t kNuBytes = CP * D * 2;
  static_assert(CP == 128 || CP == 256, "CP must be 128 or 256");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AssignSmem* S = reinterpret_cast<AssignSmem*>(base);
  uint8_t* xs = base + kAssignHeader;
  uint8_t* nuh = xs + 2 * kXBytes;
  uint8_t* nul = nuh + kNuBytes;
  uint8_t* ones = nul + kNuBytes;
  uint8_t* kparts = ones + kTileRows * kExtraK * 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = (nv + kTileRows - 1) / kTileRows;
  const long long total = static_cast<long long>(BH) * ntiles;
  const long long g0 = total * blockIdx.x / gridDim.x;
  const long long g1 = total * (blockIdx.x + 1) / gridDim.x;
  if (g0 >= g1) return;
  // the error word can change under us: decide once for the whole CTA
  if (__syncthreads_or(timed_out_before(err) ? 1 : 0)) return;

  if (tid == 0) {
    S->abort = 0;
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&S->x_full[b]), 1);
      // one arrival per warp (after __syncwarp), not per thread
      mbar_init(smem_u32(&S->x_free[b]), kScorerWarps);
      mbar_init(smem_u32(&S->t_full[b]), 1);
      mbar_init(smem_u32(&S->t_free[b]), kScorerWarps);
      mbar_init(smem_u32(&S->l_full[b]), kScorerWarps / 2);
      mbar_init(smem_u32(&S->l_free[b]), kSummerWarps);
    }
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&S->tmem_base), 2 * CP);
    tmem_relinquish();
  }
  // the A operand of the kappa chunk: ones in columns 0..2 of every row
  for (int e = tid; e < kTileRows * kExtraK; e += kAssignThreads) {
    const int row = e / kExtraK, k = e % kExtraK;
    *reinterpret_cast<uint16_t*>(ones + plain_offset(row, k)) = k < 3 ? 0x3F80 : 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;
  volatile int* abort = &S->abort;
  constexpr uint32_t idesc = idesc_bf16_f32(128, CP, false, false);

  // producer state (warp 0, lane 0)
  uint32_t tma_pend = 0;         // buffers with a TMA not yet waited on
  uint32_t tma_par[2] = {0, 0};  // x_full parity each of them completes
  int mma_last = -1;

  long long g = g0;
  int i = 0;  // tiles started by this CTA: selects buffers and barrier phases
  while (g < g1) {
    const int h = static_cast<int>(g / ntiles);
    const int t0 = static_cast<int>(g - static_cast<long long>(h) * ntiles);
    const int t1 = static_cast<int>(min(static_cast<long long>(ntiles), g1 - static_cast<long long>(h) * ntiles));
    const int row0 = h * N;
    __syncthreads();  // every role is done with the previous head
    if (*abort) break;
    {  // head h: nu_hi, nu_lo into the swizzled K-major layout of the B operand,
       // -kappa/2 in three bf16 parts into the kappa chunk, and the bound's maxima
      constexpr int chunks = D / 8;
      const uint4* srch = reinterpret_cast<const uint4*>(nu_hi + static_cast<size_t>(h) * CP * D);
      const uint4* srcl = reinterpret_cast<const uint4*>(nu_lo + static_cast<size_t>(h) * CP * D);
      for (int e = tid; e < CP * chunks; e += kAssignThreads) {
        const int j = e / chunks, c = e % chunks;
        const uint32_t off = sw128_offset(j, c * 8, CP);
        const uint4 vh = __ldg(srch + e), vl = __ldg(srcl + e);
        *reinterpret_cast<uint4*>(nuh + off) = vh;
        *reinterpret_cast<uint4*>(nul + off) = vl;
      }
      for (int j = tid; j < CP; j += kAssignThreads) {
        uint16_t p[3] = {0, 0, 0};
        if (j < C) {
          const double v = -0.5 * kappa64[h * CP + j];
          p[0] = bf16_bits_rn(static_cast<float>(v));
          const double r1 = v - static_cast<double>(__uint_as_float(static_cast<uint32_t>(p[0]) << 16));
          p[1] = bf16_bits_rn(static_cast<float>(r1));
          const double r2 = r1 - static_cast<double>(__uint_as_float(static_cast<uint32_t>(p[1]) << 16));
          p[2] = bf16_bits_rn(static_cast<float>(r2));
        } else {
          p[0] = 0xF880;  // -2^114: a padding column never wins
        }
        for (int k = 0; k < kExtraK; ++k)
          *reinterpret_cast<uint16_t*>(kparts + plain_offset(j, k)) = k < 3 ? p[k] : 0;
      }
      if (warp == 0) {
        float mn = 0.f, mk = 0.f;
        for (int j = lane; j < C; j += 32) {
          mn = fmaxf(mn, nunorm[h * CP + j]);
          mk = fmaxf(mk, static_cast<float>(fabs(kappa64[h * CP + j])));
        }
        for (int o = 16; o > 0; o >>= 1) {
          mn = fmaxf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mk = fmaxf(mk, __shfl_xor_sync(0xffffffffu, mk, o));
        }
        if (lane == 0) {
          S->max_nrm = mn;
          S->max_kap = mk;
        }
      }
      fence_proxy_async_smem();
    }
    __syncthreads();

    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        auto issue_tma = [&](int ii, int tt) -> bool {
          const int b = ii & 1;
          if (ii >= 2 && !mbar_wait(smem_u32(&S->x_free[b]), ((ii >> 1) - 1) & 1, abort)) return false;
          mbar_arrive_expect_tx(smem_u32(&S->x_full[b]), kXBytes);
          for (int s = 0; s < D / 64; ++s)
            tma_load_2d(&xmap, smem_u32(xs + b * kXBytes + s * kTileRows * 128), smem_u32(&S->x_full[b]),
                        s * 64, row0 + tt * kTileRows);
          tma_pend |= 1u << b;
          tma_par[b] = (ii >> 1) & 1;
          return true;
        };
        bool ok = issue_tma(i, t0);
        const uint32_t ha = smem_u32(nuh), la = smem_u32(nul);
        const uint64_t ad_k = plain_desc(smem_u32(ones), 128, 256);
        const uint64_t bd_k = plain_desc(smem_u32(kparts), 128, 256);
        for (int tt = t0; ok && tt < t1; ++tt) {
          const int ii = i + (tt - t0), b = ii & 1;
          if (tt + 1 < t1 && !issue_tma(ii + 1, tt + 1)) break;
          if (!mbar_wait(smem_u32(&S->x_full[b]), (ii >> 1) & 1, abort)) break;
          tma_pend &= ~(1u << b);
          if (ii >= 2 && !mbar_wait(smem_u32(&S->t_free[b]), ((ii >> 1) - 1) & 1, abort)) break;
          tc_fence_after();
          const uint32_t dt = tmem + b * CP;
          const uint32_t xa = smem_u32(xs + b * kXBytes);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int sub = kk >> 2, off = (kk & 3) * 32;
            umma_f16(dt, sw128_desc(xa + sub * kTileRows * 128 + off, 16, 1024),
                     sw128_desc(ha + sub * CP * 128 + off, 16, 1024), idesc, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int sub = kk >> 2, off = (kk & 3) * 32;
            umma_f16(dt, sw128_desc(xa + sub * kTileRows * 128 + off, 16, 1024),
                     sw128_desc(la + sub * CP * 128 + off, 16, 1024), idesc, 1);
          }
          umma_f16(dt, ad_k, bd_k, idesc, 1);
          umma_commit(smem_u32(&S->t_full[b]));
          mma_last = ii;
        }
      }
      __syncwarp();
    } else if (warp >= kFirstScorer) {
      // ------------------------------------------------------------ scorers
      const int lq = warp & 3;                   // TMEM lane quarter
      const int hf = (warp - kFirstScorer) >> 2;  // column half
      const int r = lq * 32 + lane;              // tile row
      const int pair_bar = 1 + lq;
      const uint32_t lane_base = tmem + (static_cast<uint32_t>(lq * 32) << 16);
      const float max_nrm = S->max_nrm, max_kap = S->max_kap;
      for (int tt = t0; tt < t1; ++tt) {
        const int ii = i + (tt - t0), b = ii & 1;
        const uint32_t ph = (ii >> 1) & 1;
        // the MMA of this tile (and so its X copy) is complete
        const int late = (mbar_wait(smem_u32(&S->t_full[b]), ph, abort) &&
                          mbar_wait(smem_u32(&S->x_full[b]), ph, abort)) ? 0 : 1;
        if (named_sync_or(kBarScorers, kScorers, late)) break;  // every scorer leaves together
        tc_fence_after();
        {  // |x|^2 over this half of the dimensions; then the X buffer is free
          const uint8_t* xb = xs + b * kXBytes;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int c = hf * (D / 2); c < (hf + 1) * (D / 2); c += 8) {
            const uint4 v = *reinterpret_cast<const uint4*>(xb + sw128_offset(r, c, kTileRows));
            const float f0 = __uint_as_float(v.x << 16), f1 = __uint_as_float(v.x & 0xffff0000u);
            const float f2 = __uint_as_float(v.y << 16), f3 = __uint_as_float(v.y & 0xffff0000u);
            const float f4 = __uint_as_float(v.z << 16), f5 = __uint_as_float(v.z & 0xffff0000u);
            const float f6 = __uint_as_float(v.w << 16), f7 = __uint_as_float(v.w & 0xffff0000u);
            a0 = fmaf(f0, f0, fmaf(f4, f4, a0));
            a1 = fmaf(f1, f1, fmaf(f5, f5, a1));
            a2 = fmaf(f2, f2, fmaf(f6, f6, a2));
            a3 = fmaf(f3, f3, fmaf(f7, f7, a3));
          }
          S->xq[hf][r] = (a0 + a1) + (a2 + a3);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S->x_free[b]));
        // pass 1: maximum of this half's u
        const uint32_t ta = lane_base + b * CP + hf * kHalfCols;
        float mx = -INFINITY;
#pragma unroll 1
        for (int c = 0; c < kChunks; c += 2) {  // two chunks per TMEM round trip
          float v0[32], v1[32];
          tmem_ld32f(ta + 32 * c, v0);
          tmem_ld32f(ta + 32 * (c + 1), v1);
          tmem_wait_ld_f(v0);
          tmem_wait_ld_f(v1);
          float m4[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            m4[k] = fmax3(v0[8 * k], v0[8 * k + 1], v0[8 * k + 2]);
            m4[k] = fmax3(m4[k], v0[8 * k + 3], v0[8 * k + 4]);
            m4[k] = fmax3(m4[k], v0[8 * k + 5], v0[8 * k + 6]);
            m4[k] = fmax3(m4[k], v0[8 * k + 7], v1[8 * k]);
            m4[k] = fmax3(m4[k], v1[8 * k + 1], v1[8 * k + 2]);
            m4[k] = fmax3(m4[k], v1[8 * k + 3], v1[8 * k + 4]);
            m4[k] = fmax3(m4[k], v1[8 * k + 5], v1[8 * k + 6]);
            m4[k] = fmaxf(m4[k], v1[8 * k + 7]);
          }
          mx = fmax3(mx, fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        S->mh[hf][r] = mx;
        named_sync(pair_bar, 64);
        // pass 2: candidates within 2E of the row maximum
        {
          const float U = fmaxf(S->mh[0][r], S->mh[1][r]);
          const float xn = sqrtf(S->xq[0][r] + S->xq[1][r]);
          const float thr = U - ldexpf(xn * max_nrm + 0.5f * max_kap, -12);
          int k = 0;
          int16_t cl[kHalfCand] = {0, 0, 0, 0};
#pragma unroll 1
          for (int c = 0; c < kChunks; c += 2) {
            float v0[32], v1[32];
            tmem_ld32f(ta + 32 * c, v0);
            tmem_ld32f(ta + 32 * (c + 1), v1);
            tmem_wait_ld_f(v0);
            tmem_wait_ld_f(v1);
            // eight independent partial masks per word keep the OR chains short
            uint32_t p0[8], p1[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              p0[u] = 0u;
              p1[u] = 0u;
            }
#pragma unroll
            for (int q = 0; q < 32; ++q) {
              p0[q & 7] |= (v0[q] >= thr ? 1u : 0u) << q;
              p1[q & 7] |= (v1[q] >= thr ? 1u : 0u) << q;
            }
            uint32_t bw[2] = {((p0[0] | p0[1]) | (p0[2] | p0[3])) | ((p0[4] | p0[5]) | (p0[6] | p0[7])),
                              ((p1[0] | p1[1]) | (p1[2] | p1[3])) | ((p1[4] | p1[5]) | (p1[6] | p1[7]))};
#pragma unroll
            for (int w2 = 0; w2 < 2; ++w2) {
              while (bw[w2]) {
                const int q = __ffs(bw[w2]) - 1;
                bw[w2] &= bw[w2] - 1;
                if (k < kHalfCand) cl[k] = static_cast<int16_t>(hf * kHalfCols + 32 * (c + w2) + q);
                ++k;
              }
            }
          }
          S->kc[hf][r] = static_cast<uint8_t>(min(k, 255));
#pragma unroll
          for (int q = 0; q < kHalfCand; ++q) S->cand[hf][r][q] = cl[q];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S->t_free[b]));
        named_sync(pair_bar, 64);
        // the row's decision, published for the summers
        if (hf == 0) {
          if (ii >= 2) mbar_wait(smem_u32(&S->l_free[b]), ((ii >> 1) - 1) & 1, abort);
          const int tok = tt * kTileRows + r;
          int L = -1;
          if (tok < nv) {
            const int k0 = S->kc[0][r], k1 = S->kc[1][r];
            if (k0 + k1 == 1) L = k0 ? S->cand[0][r][0] : S->cand[1][r][0];
            if (k0 + k1 != 1 || L >= C) {  // (a padding column only with non-finite input)
              L = -2;
              // candidates in ascending j, unless there are too many or one
              // is a padding column (only with non-finite input)
              bool listed = k0 + k1 >= 2 && k0 <= kHalfCand && k1 <= kHalfCand;
              int n = 0;
              if (listed) {
                for (int u = 0; u < k0; ++u) S->def_cand[b][r][n++] = S->cand[0][r][u];
                for (int u = 0; u < k1; ++u) S->def_cand[b][r][n++] = S->cand[1][r][u];
                for (int u = 0; u < n; ++u) listed = listed && S->def_cand[b][r][u] < C;
              }
              S->def_n[b][r] = static_cast<int8_t>(listed ? n : 0);
            } else {
              assign[static_cast<size_t>(h) * nv + tok] = L;
            }
          }
          S->lab[b][r] = static_cast<int16_t>(L);
          // one word per 32 rows: the hf == 0 warps own rows 32 lq .. 32 lq + 31
          const uint32_t dm = __ballot_sync(0xffffffffu, L == -2);
          if (lane == 0) S->defmask[b][lq] = dm;
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&S->l_full[b]));
        }
      }
    } else {
      // ------------------------------------------------------------ summers
      // warp sw owns the contiguous rows [r0, r1) of every tile; all of them
      // are fetched with one batch of loads, one tile ahead
      const int sw = warp - kFirstSummer;
      const int r0 = kTileRows * sw / kSummerWarps, r1 = kTileRows * (sw + 1) / kSummerWarps;
      const int nr = r1 - r0;
      const float max_nrm = S->max_nrm, max_kap = S->max_kap;
      uint32_t wa0[kSumRows], wb0[kSumRows];
      auto fetch = [&](int tt, uint32_t(&wa)[kSumRows], uint32_t(&wb)[kSumRows]) {
        const uint16_t* xt = x + (static_cast<size_t>(row0) + static_cast<size_t>(tt) * kTileRows) * D;
#pragma unroll
        for (int k = 0; k < kSumRows; ++k) {
          wa[k] = 0u;
          wb[k] = 0u;
          if (k < nr && tt * kTileRows + r0 + k < nv) {
            const uint16_t* src = xt + static_cast<size_t>(r0 + k) * D;
            if (D == 128) {
              const uint2 v = __ldg(reinterpret_cast<const uint2*>(src) + lane);
              wa[k] = v.x;
              wb[k] = v.y;
            } else {
              wa[k] = __ldg(reinterpret_cast<const uint32_t*>(src) + lane);
            }
          }
        }
      };
      auto process = [&](int tt, const uint32_t(&wa)[kSumRows], const uint32_t(&wb)[kSumRows]) -> bool {
        const int ii = i + (tt - t0), b = ii & 1;
        if (!mbar_wait(smem_u32(&S->l_full[b]), (ii >> 1) & 1, abort)) return false;
        // labelled rows: a run of equal labels (token order) is summed in fp32
        // and added once to the member sums
        {
          int cur = -1, run = 0;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
          auto flush = [&]() {
            flush_row<D>(sums + (static_cast<size_t>(h) * C + cur) * D, a0, a1, a2, a3, lane);
            if (lane == 0) atomicAdd(&counts[h * C + cur], run);
          };
#pragma unroll
          for (int k = 0; k < kSumRows; ++k) {
            const int L = k < nr ? S->lab[b][r0 + k] : -1;
            if (L < 0) continue;
            if (L != cur) {
              if (cur >= 0) flush();
              cur = L;
              run = 0;
              a0 = a1 = a2 = a3 = 0.f;
            }
            ++run;
            a0 += __uint_as_float(wa[k] << 16);
            a1 += __uint_as_float(wa[k] & 0xffff0000u);
            if (D == 128) {
              a2 += __uint_as_float(wb[k] << 16);
              a3 += __uint_as_float(wb[k] & 0xffff0000u);
            }
          }
          if (cur >= 0) flush();
        }
        // deferred rows (usually none: the scorers' bitmask says which)
        const uint64_t dm64 = (static_cast<uint64_t>(S->defmask[b][(r0 >> 5) + 1 < kTileRows / 32 ? (r0 >> 5) + 1 : (r0 >> 5)]) << 32) |
                              S->defmask[b][r0 >> 5];
        uint32_t mine = static_cast<uint32_t>(dm64 >> (r0 & 31)) & ((nr >= 32 ? 0u : (1u << nr)) - 1u);
#pragma unroll 1
        while (mine) {
          const int k = __ffs(mine) - 1;
          mine &= mine - 1;
          const int rr = r0 + k;
          uint32_t xa = 0u, xb = 0u;  // this row's words (a dynamic pick from the batch)
#pragma unroll
          for (int q = 0; q < kSumRows; ++q)
            if (q == k) {
              xa = wa[q];
              xb = wb[q];
            }
          const int bj = decide_deferred<D, CP>(S, b, rr, xa, xb, nuh, nul, kparts, max_nrm, max_kap,
                                                nu64 + static_cast<size_t>(h) * C * D,
                                                kappa64 + static_cast<size_t>(h) * CP, C, lane);
          if (lane == 0) {
            assign[static_cast<size_t>(h) * nv + tt * kTileRows + rr] = bj;
            atomicAdd(&counts[h * C + bj], 1);
          }
          flush_row<D>(sums + (static_cast<size_t>(h) * C + bj) * D, __uint_as_float(xa << 16),
                       __uint_as_float(xa & 0xffff0000u), __uint_as_float(xb << 16),
                       __uint_as_float(xb & 0xffff0000u), lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S->l_free[b]));
        return true;
      };
      if (t0 < t1) fetch(t0, wa0, wb0);
      for (int tt = t0; tt < t1; ++tt) {
        if (!process(tt, wa0, wb0)) break;
        if (tt + 1 < t1) fetch(tt + 1, wa0, wb0);
      }
    }
    i += t1 - t0;
    g += t1 - t0;
  }
  __syncthreads();
  if (*abort && tid == 0) {
    report_error(err, kErrTimeoutCluster);
    // copies and MMAs still in flight complete before the buffers go away
    volatile int keep_waiting = 0;
    for (int b = 0; b < 2; ++b)
      if (tma_pend & (1u << b)) mbar_wait(smem_u32(&S->x_full[b]), tma_par[b], &keep_waiting);
    if (mma_last >= 0) mbar_wait(smem_u32(&S->t_full[mma_last & 1]), (mma_last >> 1) & 1, &keep_waiting);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 2 * CP);
}

// ---------------------------------------------------------------- finalize

// grid (C, BH), block d.
__global__ void finalize_kernel(float* __restrict__ sums, int32_t* __restrict__ counts,
                                float* __restrict__ cent, int32_t* __restrict__ sizes, int C,
                                int d) {
  const int h = blockIdx.y, j = blockIdx.x, i = threadIdx.x;
  const int n = counts[h * C + j];
  const size_t o = (static_cast<size_t>(h) * C + j) * d + i;
  if (n > 0) cent[o] = static_cast<float>(static_cast<double>(sums[o]) / static_cast<double>(n));
  sums[o] = 0.f;
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
  uint16_t* nu_hi;
  uint16_t* nu_lo;
  double* kappa64;
  float* kappa;
  float* nunorm;
  float* sums;
  int32_t* counts;
};

// columns of the scoring MMA: the cluster count padded so that four threads
// per row read one or two 32-column TMEM chunks each
inline int score_cols(int c) { return c <= 128 ? 128 : 256; }

size_t carve_step(void* ws, int BH, int d, int Cmax, StepWs* out) {
  Carver cv(ws);
  const int CP = score_cols(Cmax);
  StepWs w;
  w.M = cv.take<double>(static_cast<size_t>(BH) * d * d);
  w.nu64 = cv.take<double>(static_cast<size_t>(BH) * Cmax * d);
  w.nu_hi = cv.take<uint16_t>(static_cast<size_t>(BH) * CP * d);
  w.nu_lo = cv.take<uint16_t>(static_cast<size_t>(BH) * CP * d);
  w.kappa64 = cv.take<double>(static_cast<size_t>(BH) * CP);
  w.kappa = cv.take<float>(static_cast<size_t>(BH) * CP);
  w.nunorm = cv.take<float>(static_cast<size_t>(BH) * CP);
  w.sums = cv.take<float>(static_cast<size_t>(BH) * Cmax * d);
  w.counts = cv.take<int32_t>(static_cast<size_t>(BH) * Cmax);
  if (out) *out = w;
  return cv.used + 256;
}

template <int D, int CP>
svoo_status launch_assign(const CUtensorMap& xmap, const svoo_shape* sh, const void* x, int C,
                          const StepWs& w, int32_t* assign, int32_t* dev_err, cudaStream_t st) {
  const int BH = bh_of(sh), N = sh->N, nv = nvideo_of(sh);
  const size_t smem = 1024 + kAssignHeader + 2 * static_cast<size_t>(kTileRows) * D * 2 +
                      2 * static_cast<size_t>(CP) * D * 2 + (kTileRows + CP) * kExtraK * 2;
  if (cudaFuncSetAttribute(assign_kernel<D, CP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SVOO_ERR_CUDA;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SVOO_ERR_CUDA;
  const long long total = static_cast<long long>(BH) * ((nv + kTileRows - 1) / kTileRows);
  const int grid = static_cast<int>(total < sms ? total : sms);
  assign_kernel<D, CP><<<grid, kAssignThreads, smem, st>>>(
      xmap, static_cast<const uint16_t*>(x), N, nv, C, BH, w.nu_hi, w.nu_lo, w.nu64, w.kappa64,
      w.nunorm, assign, w.sums, w.counts, dev_err);
  return SVOO_OK;
}

// One half-step. metric_cent == nullptr: identity metric.
svoo_status run_step(const svoo_shape* sh, const void* x, int C, float* cent, int32_t* sizes,
                     int32_t* assign, const float* metric_cent, const int32_t* metric_sizes,
                     int metric_C, const StepWs& w, int32_t* dev_err, cudaStream_t st,
                     int zero_C) {
  const int BH = bh_of(sh), d = sh->d, N = sh->N;
  const int CP = score_cols(C);
  // finalize_kernel re-zeroes what a step used, so only the first step of a
  // call clears the accumulators (for the largest cluster count of the call).
  if (zero_C > 0) {
    if (cudaMemsetAsync(w.sums, 0, sizeof(float) * BH * static_cast<size_t>(zero_C) * d, st) != cudaSuccess ||
        cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * BH * static_cast<size_t>(zero_C), st) != cudaSuccess)
      return SVOO_ERR_CUDA;
  }
  if (metric_cent) {
    const int T = d / kMBlk;
    if (cudaFuncSetAttribute(metric_m_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kMetricMSmem)) != cudaSuccess)
      return SVOO_ERR_CUDA;
    metric_m_kernel<<<dim3(T * (T + 1) / 2, BH), kMThreads, kMetricMSmem, st>>>(metric_cent, metric_sizes,
                                                                                metric_C, d, w.M);
  }
  if (cudaFuncSetAttribute(metric_nu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(metric_nu_smem(d))) != cudaSuccess)
    return SVOO_ERR_CUDA;
  metric_nu_kernel<<<dim3(CP / 32, BH), 128, metric_nu_smem(d), st>>>(
      metric_cent ? w.M : nullptr, cent, C, CP, d, w.nu64, w.nu_hi, w.nu_lo, w.kappa64, w.kappa,
      w.nunorm);
  CUtensorMap xmap;
  if (encode_tiled_2d(&xmap, x, static_cast<uint64_t>(BH) * N, d, kTileRows, 64) != CUDA_SUCCESS)
    return SVOO_ERR_CUDA;
  svoo_status s;
  if (d == 128)
    s = CP == 256 ? launch_assign<128, 256>(xmap, sh, x, C, w, assign, dev_err, st)
                  : launch_assign<128, 128>(xmap, sh, x, C, w, assign, dev_err, st);
  else
    s = CP == 256 ? launch_assign<64, 256>(xmap, sh, x, C, w, assign, dev_err, st)
                  : launch_assign<64, 128>(xmap, sh, x, C, w, assign, dev_err, st);
  if (s != SVOO_OK) return s;
  finalize_kernel<<<dim3(C, BH), d, 0, st>>>(w.sums, w.counts, cent, sizes, C, d);
  return launch_status();
}

bool cluster_counts_ok(int C) { return C >= 1 && C <= 256; }

// Cluster count that sizes a half-step's scratch: metric_C only counts when a
// metric is given (it is ignored, whatever its value, for the identity).
int step_clusters(int C, const float* metric_cent, int metric_C) {
  return (metric_cent && metric_C > C) ? metric_C : C;
}

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
  size_t need = carve_step(workspace, BH, shape->d, step_clusters(C, metric_cent, metric_C), &w);
  if (workspace_bytes < need) return SVOO_ERR_WORKSPACE;
  return run_step(shape, x, C, cent, sizes, assign, metric_cent, metric_sizes, metric_C, w, dev_err,
                  static_cast<cudaStream_t>(stream), C);
}

extern "C" svoo_status svoo_cluster(const svoo_shape* shape, const void* q, const void* k, int n_qc,
                                    int n_kc, int iters, int flags, int32_t* q_assign,
                                    int32_t* k_assign, float* q_cent, float* k_cent,
                                    int32_t* q_sizes, int32_t* k_sizes, void* workspace,
                                    size_t workspace_bytes, int32_t* dev_err, void* stream) {
  if (!shape_ok(shape) || !q || !k || !q_assign || !k_assign || !q_cent || !k_cent || !q_sizes ||
      !k_sizes || !workspace)
    return SVOO_ERR_INVALID_ARG;
  if (!cluster_counts_ok(n_qc) || !cluster_counts_ok(n_kc) || iters < 1 ||
      (flags & ~(SVOO_CLUSTER_WARM | SVOO_CLUSTER_IDENTITY)) != 0)
    return SVOO_ERR_INVALID_ARG;
  const bool warm = (flags & SVOO_CLUSTER_WARM) != 0;
  const bool identity = (flags & SVOO_CLUSTER_IDENTITY) != 0;
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
    const bool ident = identity || (it == 0 && !warm);
    svoo_status s = run_step(shape, q, n_qc, q_cent, q_sizes, q_assign, ident ? nullptr : k_cent,
                             k_sizes, n_kc, w, dev_err, st, it == 0 ? Cmax : 0);
    if (s != SVOO_OK) return s;
    s = run_step(shape, k, n_kc, k_cent, k_sizes, k_assign, identity ? nullptr : q_cent, q_sizes,
                 n_qc, w, dev_err, st, 0);
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
  const int Cmax = step_clusters(C, metric_cent, metric_C);
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
