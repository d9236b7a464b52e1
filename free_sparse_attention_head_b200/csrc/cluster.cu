// cluster.cu -- per-head bidirectional QK co-clustering (SVOO abstract; iCATS
// sections 3.1 and 4.1): k-means of the query tokens and of the key tokens,
// each side's distance being the interaction error under the metric of the
// other side's clusters, M = sum_b n_b c_b c_b^T / sum_b n_b (identity in the
// cold first query step).
//
// Kernels of one half-step (one side):
//   metric_m_kernel   M from the other side's centroids and sizes (fp64)
//   metric_nu_kernel  nu_j = M mu_j, kappa_j = mu_j . nu_j (fp64), nu_j split
//                     into two bf16 rows (hi + lo), -kappa_j/2 in three bf16
//                     parts, and per-block maxima of |nu_j|, |kappa_j| for the bound
//   xnorm_kernel      |x|^2 of every token, once per side and call (the
//                     assignment's error bound)
//   assign_kernel     persistent, warp-specialised, dynamically scheduled
//                     stream of 128-token tiles: tcgen05 MMAs against
//                     [nu_hi | nu_lo | kappa] into double-buffered TMEM; per
//                     token the score kappa_j - 2 x.nu_j is bounded by the
//                     MMA error and a token with a single candidate takes it
//   fixup_kernel      the other tokens, exactly in fp64: their listed
//                     candidates, or every cluster (ties to the smaller j)
//   update_kernel     member sums in fp64, exact (so order-independent), per
//                     chunk of consecutive tokens grouped by label; within a
//                     call, after each side's first half-step, only the tokens
//                     whose label changed move between the kept sums
//   finalize_kernel   centroid = fp32(sum / count), empty clusters keep
//                     theirs; resets the chunk counters (and a lone
//                     half-step's sums).
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
__host__ __device__ __forceinline__ uint32_t plain_offset(int row, int k) {
  return static_cast<uint32_t>((row >> 3) * 256 + (k >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2);
}

__device__ __forceinline__ uint16_t bf16_bits_rn(float f) {
  const __nv_bfloat16 b = __float2bfloat16_rn(f);
  return *reinterpret_cast<const uint16_t*>(&b);
}

// -kappa/2 as three bf16 parts whose sum equals it to 2^-26 relative; a
// padding column gets -2^114 and never wins
__device__ __forceinline__ void kappa_parts(double kappa, bool real, uint16_t (&p)[3]) {
  p[0] = p[1] = p[2] = 0;
  if (!real) {
    p[0] = 0xF880;
    return;
  }
  const double v = -0.5 * kappa;
  p[0] = bf16_bits_rn(static_cast<float>(v));
  const double r1 = v - static_cast<double>(__uint_as_float(static_cast<uint32_t>(p[0]) << 16));
  p[1] = bf16_bits_rn(static_cast<float>(r1));
  const double r2 = r1 - static_cast<double>(__uint_as_float(static_cast<uint32_t>(p[1]) << 16));
  p[2] = bf16_bits_rn(static_cast<float>(r2));
}

// nu_j = M mu_j and kappa_j = mu_j . nu_j in fp64; nu_j also as the pair of
// bf16 rows nu_hi = bf16(nu_j), nu_lo = bf16(nu_j - nu_hi) that the scoring
// MMA consumes (their sum is nu_j to 2^-18 relative). Clusters j
// in [C, CP) are padding (nu = 0, kappa = +inf). grid (CP/kNuCl, BH), block
// 128: warp w owns clusters j0 + 4w .. +3, lane owns dimensions 2 lane, 2 lane + 1
// (and 64 + the same for d = 128). Rows of M arrive 16 at a time by cp.async,
// one chunk ahead. M == nullptr means the identity. For the scoring MMA it
// also writes, per head, the kappa parts tile (-kappa_j/2 in three bf16
// parts, rows j of a [CP][16] tile in the no-swizzle core-matrix layout,
// exactly as it lies in shared memory) and, per block of kNuCl clusters,
// (max |nu_j|, max |kappa_j|) over its real clusters.
constexpr int kNuRows = 16;
constexpr int kNuCl = 16;            // clusters per block
constexpr int kNuWarpCl = kNuCl / 4;  // clusters per warp
constexpr int kExtraK = 16;  // K width of the kappa chunk of the scoring MMA
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
                     uint16_t* __restrict__ kimg,
                     float2* __restrict__ numax) {
  extern __shared__ __align__(16) double nsm[];
  __shared__ float2 wmax[4];
  double* mu = nsm;                          // [kNuCl][kNuMuStride]
  double* mch = mu + kNuCl * kNuMuStride;    // two buffers of [16][d]
  const int h = blockIdx.y, j0 = blockIdx.x * kNuCl;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const double* Mh = M ? M + static_cast<size_t>(h) * d * d : nullptr;
  auto stage = [&](int chunk) {  // rows 16 chunk .. +15 of M into buffer chunk % 2
    double* dst = mch + (chunk & 1) * kNuRows * d;
    const double* src = Mh + static_cast<size_t>(chunk) * kNuRows * d;
    for (int e = threadIdx.x; e < kNuRows * d / 2; e += blockDim.x) cp_async16(dst + 2 * e, src + 2 * e);
    cp_async_commit();
  };
  if (Mh) stage(0);
  {  // the block's centroids, all float4 loads in flight before any store
    constexpr int kLd = kNuCl * 128 / 4 / 128;  // float4 per thread (d = 128; half of them for d = 64)
    float4 f[kLd];
#pragma unroll
    for (int q = 0; q < kLd; ++q) {
      const int e = (threadIdx.x + q * 128) * 4, r = e / d, c = e % d;
      f[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (e < kNuCl * d && j0 + r < C)
        f[q] = __ldg(reinterpret_cast<const float4*>(cent + (static_cast<size_t>(h) * C + j0 + r) * d + c));
    }
#pragma unroll
    for (int q = 0; q < kLd; ++q) {
      const int e = (threadIdx.x + q * 128) * 4, r = e / d, c = e % d;
      if (e < kNuCl * d) {
        double* m = mu + r * kNuMuStride + c;
        m[0] = f[q].x;
        m[1] = f[q].y;
        m[2] = f[q].z;
        m[3] = f[q].w;
      }
    }
  }
  const int nd = d == 128 ? 4 : 2;  // dimensions per lane
  const int dim[4] = {2 * lane, 2 * lane + 1, 64 + 2 * lane, 65 + 2 * lane};
  const double* mw = mu + kNuWarpCl * warp * kNuMuStride;
  double acc[kNuWarpCl][4];  // [cluster][dimension]
#pragma unroll
  for (int u = 0; u < kNuWarpCl; ++u)
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
        for (int u = 0; u < kNuWarpCl; ++u) {
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
    for (int u = 0; u < kNuWarpCl; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = v < nd ? mw[u * kNuMuStride + dim[v]] : 0.0;
  }
  float mx_n = 0.f, mx_k = 0.f;
#pragma unroll
  for (int u = 0; u < kNuWarpCl; ++u) {
    const int j = j0 + kNuWarpCl * warp + u;
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
      const float nn = j < C ? static_cast<float>(sqrt(k2)) : 0.f;
      kappa64[h * CP + j] = j < C ? k1 : INFINITY;
      uint16_t p[3];
      kappa_parts(k1, j < C, p);
      uint8_t* img = reinterpret_cast<uint8_t*>(kimg + static_cast<size_t>(h) * CP * kExtraK);
      *reinterpret_cast<uint4*>(img + plain_offset(j, 0)) =
          make_uint4(p[0] | (static_cast<uint32_t>(p[1]) << 16), p[2], 0u, 0u);
      *reinterpret_cast<uint4*>(img + plain_offset(j, 8)) = make_uint4(0u, 0u, 0u, 0u);
      if (j < C) {
        mx_n = fmaxf(mx_n, nn);
        mx_k = fmaxf(mx_k, static_cast<float>(fabs(k1)));
      }
    }
  }
  if (lane == 0) wmax[warp] = make_float2(mx_n, mx_k);
  __syncthreads();
  if (threadIdx.x == 0) {
    float2 m = wmax[0];
    for (int w = 1; w < 4; ++w) m = make_float2(fmaxf(m.x, wmax[w].x), fmaxf(m.y, wmax[w].y));
    numax[h * (CP / kNuCl) + blockIdx.x] = m;
  }
}
inline size_t metric_nu_smem(int d) { return (kNuCl * kNuMuStride + 2 * kNuRows * d) * sizeof(double); }

// ---------------------------------------------------------------- assign
//
// Persistent, warp-specialised kernel, one CTA per SM, over a stream of
// 128-token tiles. The (head, tile) space is handed out in chunks of
// kChunkTiles tiles of one head through per-head counters: a CTA starts at its
// own head and moves on to the next head with chunks left, so SMs that run
// this kernel faster take more chunks (on B200 some SMs ran the same tiles up
// to 1.5x slower than others, so a static split left the fast ones idle).
// Tile i of a CTA uses TMEM accumulator i % 2 (CP fp32 columns); its X rows
// arrive in d/64 stages (128 x 64 bf16, one TMA box each) of a ring of
// kStages, and a stage goes back to the ring when the MMAs that read it are
// done (a tcgen05 commit), so copies run two tiles ahead of the MMAs.
//   scheduler (warp 17) claims the CTA's next chunk while the current one
//                       runs (one chunk ahead); its lanes probe 32 head
//                       counters at a time.
//   producer (warp 0)   streams the chunks' tiles: TMA of the X stages two
//                       tiles ahead; per tile, once its accumulator is free,
//                       publishes the tile's head and index for the scorers;
//                       on a head change, once the tensor cores are done with
//                       the old head, TMA of the new head's nu_hi, nu_lo and
//                       kappa parts; then one tcgen05 chain per tile:
//                       u = X . nu_hi^T + X . nu_lo^T + 1 . (-kappa/2)^T, the
//                       last term a 16-wide K chunk of ones against -kappa_j/2
//                       split into three bf16 parts, so u_j = x.nu_j - kappa_j/2
//                       and the score is kappa_j - 2 x.nu_j = -2 u_j.
//   scorers (warps 1-16) never read X (|x|^2 comes from xnorm_kernel); warp w
//                       reads TMEM lane quarter w % 4 (32 rows) and
//                       column quarter (w - 1) / 4: each thread loads its row's
//                       CP/4 scores into registers (then the accumulator goes
//                       back) and takes the quarter's maximum; the four
//                       quarters of a row meet in shared memory for the row
//                       maximum U and the error bound E; each thread finds its
//                       quarter's candidates u_j >= U - 2E (together they
//                       contain the exact argmin of the score) and publishes
//                       their count. From the four counts the four warps take
//                       the same decision for the row: one candidate is the
//                       label, written by the warp that holds it; up to
//                       kDeferCand (at most kQuarterCand from each quarter)
//                       are listed for the row in its 32-row group's record,
//                       each warp writing its own; more, or none at all (only
//                       with non-finite input), give label -2, every
//                       cluster. fixup_kernel decides the listed and -2 rows.
//
// Error bound: nu_hi + nu_lo equals nu to 2^-18 relative and the three kappa
// parts give kappa to 2^-26; the MMA's fp32 accumulation of 2d + 3 exact
// products adds at most (2d + 3) 2^-23 of the sum of their magnitudes, at most
// |x||nu_j| (1 + 2^-8) + |kappa_j| / 2. E = 2^-13 (|x| max|nu| + max|kappa| / 2)
// bounds |u_computed - u| with a factor of two to spare.

// |x|^2 of the video tokens of every head (fp32 [BH][nv]), read by the
// scorers for the error bound. grid (ceil(nv / 32), BH), block 256: a warp
// takes 4 rows at a time, lane l holding dimensions (D/32) l .. (D/32) l + D/32 - 1.
template <int D>
__global__ void __launch_bounds__(256)
    xnorm_kernel(const uint16_t* __restrict__ x, int N, int nv, float* __restrict__ xnorm) {
  constexpr int kPer = D / 32;
  const int h = blockIdx.y, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r0 = blockIdx.x * 32 + warp * 4;
  float s[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    s[q] = 0.f;
    const int r = r0 + q;
    if (r < nv) {
      const uint16_t* row = x + (static_cast<size_t>(h) * N + r) * D;
      if constexpr (kPer == 4) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(row) + lane);
        const float a = __uint_as_float(w.x << 16), b = __uint_as_float(w.x & 0xffff0000u);
        const float c = __uint_as_float(w.y << 16), d = __uint_as_float(w.y & 0xffff0000u);
        s[q] = fmaf(a, a, b * b) + fmaf(c, c, d * d);
      } else {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(row) + lane);
        const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xffff0000u);
        s[q] = fmaf(a, a, b * b);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int q = 0; q < 4; ++q) s[q] += __shfl_xor_sync(0xffffffffu, s[q], o);
  if (lane < 4 && r0 + lane < nv) {
    float v = s[0];
#pragma unroll
    for (int q = 1; q < 4; ++q)
      if (lane == q) v = s[q];
    xnorm[static_cast<size_t>(h) * nv + r0 + lane] = v;
  }
}

constexpr int kScorerWarps = 16;
constexpr int kSchedWarp = 1 + kScorerWarps;
constexpr int kAssignWarps = 2 + kScorerWarps;
constexpr int kAssignThreads = kAssignWarps * 32;
constexpr int kTileRows = 128;
constexpr int kStages = 5;              // X ring: 128-row x 64-column (16 KB) stages
constexpr int kStageBytes = kTileRows * 64 * 2;
constexpr int kQuarterCand = 16;     // candidates a quarter may add to a listed row
constexpr int kDeferCand = 32;       // candidates of a listed row
constexpr int kDeferAll = 1 << 8;    // defer_count flag: some rows of the group have label -2
constexpr int kChunkTiles = 4;       // tiles per claimed chunk
constexpr int kAssignHeader = 4096;  // AssignSmem, keeps the X stages 1024-aligned

// The rows of one 32-row group (a TMEM lane quarter of one tile) that have
// several candidates, decided by fixup_kernel: row l's count (0: not listed)
// and its candidates, ascending (cluster ids, < 256).
struct DeferGroup {
  uint8_t n[32];
  uint8_t cand[32][kDeferCand];
};

struct AssignSmem {
  uint64_t xs_full[kStages], xs_free[kStages];  // X stages: TMA landed / the MMAs reading it are done
  uint64_t t_full[2], t_free[2];                // TMEM accumulators: MMA done / scores read
  uint64_t info_full[2];                        // the accumulator's tile (head, index) is published
  uint64_t nu_full, sched_full, sched_free;
#ifdef SVOO_TEST_STALL
  uint64_t stall;  // test-only: a barrier that nothing completes
#endif
  uint32_t tmem_base;
  int abort;
  int tile_h[2], tile_t[2];  // head and tile of each accumulator's tile (head -1: the end)
  int sched_h, sched_c;      // the scheduler's claimed chunk (head -1: none left)
  float mq[4][kTileRows];    // per-quarter maxima of u
  uint32_t kc[kTileRows];    // candidates per column quarter, a byte each (saturating)
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

// untiled bulk copy global -> shared, completing on `bar` (bytes; 16-byte
// aligned addresses and size)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// bit (q) of m set where v >= thr: a compare and a predicated OR per value
__device__ __forceinline__ void mark_ge(uint32_t& m, float v, float thr, uint32_t bit) {
  asm("{\n\t.reg .pred p;\n\t"
      "setp.ge.f32 p, %1, %2;\n\t"
      "@p or.b32 %0, %0, %3;\n\t}"
      : "+r"(m)
      : "f"(v), "f"(thr), "r"(bit));
}

// grid: min(#SMs, chunks) CTAs, block kAssignThreads. Dynamic smem:
// [AssignSmem][X kStages x 128 x 64 bf16][nu_hi CP x D][nu_lo CP x D][ones 128 x 16][kappa parts CP x 16]
// kimg: per head the kappa parts tile as it lies in shared memory; numax: per
// head and kNuCl-cluster block, (max |nu_j|, max |kappa_j|); xnorm: |x|^2 of the
// tokens (xnorm_kernel).
template <int D, int CP>
__global__ void __launch_bounds__(kAssignThreads, 1)
    assign_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap himap,
                  const __grid_constant__ CUtensorMap lomap, int N, int nv, int C, int BH,
                  const uint16_t* __restrict__ kimg, const float2* __restrict__ numax,
                  int32_t* __restrict__ head_next, int32_t* __restrict__ assign,
                  int32_t* __restrict__ defer_count, DeferGroup* __restrict__ defer,
                  const float* __restrict__ xnorm, int* __restrict__ err) {
  constexpr int kQCols = CP / 4;      // score columns per scorer thread
  constexpr int kLoads = kQCols / 32;  // 32-column TMEM loads per thread
  constexpr int kSpt = D / 64;         // X stages per tile
  constexpr uint32_t kNuBytes = CP * D * 2;
  constexpr uint32_t kKBytes = CP * kExtraK * 2;
  static_assert(CP == 128 || CP == 256, "CP must be 128 or 256");
  static_assert(kSpt >= 1 && 2 * kSpt < kStages, "the ring holds two tiles ahead");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AssignSmem* S = reinterpret_cast<AssignSmem*>(base);
  uint8_t* xs = base + kAssignHeader;
  uint8_t* nuh = xs + kStages * kStageBytes;
  uint8_t* nul = nuh + kNuBytes;
  uint8_t* ones = nul + kNuBytes;
  uint8_t* kparts = ones + kTileRows * kExtraK * 2;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = (nv + kTileRows - 1) / kTileRows;
  const int nchunk = (ntiles + kChunkTiles - 1) / kChunkTiles;
  // the error word can change under us: decide once for the whole CTA
  if (__syncthreads_or(timed_out_before(err) ? 1 : 0)) return;

  if (tid == 0) {
    S->abort = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_u32(&S->xs_full[s]), 1);
      mbar_init(smem_u32(&S->xs_free[s]), 1);  // a tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&S->t_full[b]), 1);
      // one arrival per warp (after __syncwarp), not per thread
      mbar_init(smem_u32(&S->t_free[b]), kScorerWarps);
      mbar_init(smem_u32(&S->info_full[b]), 1);
    }
    mbar_init(smem_u32(&S->nu_full), 1);
    mbar_init(smem_u32(&S->sched_full), 1);
    mbar_init(smem_u32(&S->sched_free), 1);
#ifdef SVOO_TEST_STALL
    mbar_init(smem_u32(&S->stall), 1);
#endif
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&himap);
    tma_prefetch_desc(&lomap);
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
  fence_proxy_async_smem();  // read by the tensor cores
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S->tmem_base;
  volatile int* abort = &S->abort;
  constexpr uint32_t idesc = idesc_bf16_f32(128, CP, false, false);

  // producer state (warp 0, lane 0), also read by the abort path below
  uint32_t xs_pend = 0;             // X stages with a TMA not yet waited on
  uint32_t xs_par[kStages] = {};    // xs_full parity each of them completes
  int mma_last = -1;
  bool nu_pend = false;             // operand copy not yet waited on
  uint32_t nu_par = 0;              // nu_full parity of the next operand copy

  if (warp == kSchedWarp) {
    // ------------------------------------------------------------ scheduler
    int h_from = static_cast<int>(static_cast<long long>(blockIdx.x) * BH / gridDim.x);
    for (int n = 0;; ++n) {
      int ok = 1;
      if (lane == 0 && n >= 1) ok = mbar_wait(smem_u32(&S->sched_free), (n - 1) & 1, abort) ? 1 : 0;
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      int found = -1, c = 0;
      // heads h_from, h_from + 1, ... (cyclically), 32 at a time; a head whose
      // counter has run out stays so, so every try that fails ends a head
      for (int k0 = 0; k0 < BH && found < 0; k0 += 32) {
        const int k = k0 + lane;
        const int hh = h_from + k < BH ? h_from + k : h_from + k - BH;
        const int open = (k < BH && *reinterpret_cast<volatile int32_t*>(head_next + hh) < nchunk) ? 1 : 0;
        unsigned m = __ballot_sync(0xffffffffu, open);
        while (m && found < 0) {
          const int l = __ffs(m) - 1;
          m &= m - 1;
          int got = 0;
          if (lane == l) got = atomicAdd(&head_next[hh], 1);
          got = __shfl_sync(0xffffffffu, got, l);
          const int hl = __shfl_sync(0xffffffffu, hh, l);
          if (got < nchunk) {
            found = hl;
            c = got;
          }
        }
      }
      if (found >= 0) h_from = found;
      if (lane == 0) {
        S->sched_h = found;
        S->sched_c = c;
        mbar_arrive(smem_u32(&S->sched_full));
      }
      if (found < 0) break;
    }
  } else if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int n_pop = 0, ch = -1, ct = 0, ce = 0;  // current chunk: head, next tile, end
      int th[4], tti[4];                       // head and tile of the stream's tiles ii (mod 4)
      int known = 0;                           // tiles of the stream known so far
      bool ended = false;
      // learn tiles up to index want; false on a timeout
      auto fetch = [&](int want) -> bool {
        while (!ended && known <= want) {
          if (ct >= ce) {
            if (!mbar_wait(smem_u32(&S->sched_full), n_pop & 1, abort)) return false;
            ch = S->sched_h;
            const int c = S->sched_c;
            mbar_arrive(smem_u32(&S->sched_free));
            ++n_pop;
            if (ch < 0) {
              ended = true;
              break;
            }
            ct = c * kChunkTiles;
            ce = min(ntiles, ct + kChunkTiles);
          }
          th[known & 3] = ch;
          tti[known & 3] = ct++;
          ++known;
        }
        return true;
      };
      // TMA of tile ii's X stages (ring slot of stage q: q % kStages; its
      // previous occupant, stage q - kStages, is released by an MMA commit)
      auto load_tile = [&](int ii) -> bool {
        for (int s = 0; s < kSpt; ++s) {
          const int q = ii * kSpt + s, slot = q % kStages, use = q / kStages;
          if (use >= 1 && !mbar_wait(smem_u32(&S->xs_free[slot]), (use - 1) & 1, abort)) return false;
          mbar_arrive_expect_tx(smem_u32(&S->xs_full[slot]), kStageBytes);
          tma_load_2d(&xmap, smem_u32(xs + slot * kStageBytes), smem_u32(&S->xs_full[slot]), s * 64,
                      th[ii & 3] * N + tti[ii & 3] * kTileRows);
          xs_pend |= 1u << slot;
          xs_par[slot] = use & 1;
        }
        return true;
      };
      // head h's MMA operands, once the tensor cores are done with the old ones
      auto load_nu = [&](int h) -> bool {
        if (mma_last >= 0 && !mbar_wait(smem_u32(&S->t_full[mma_last & 1]), (mma_last >> 1) & 1, abort))
          return false;
        mbar_arrive_expect_tx(smem_u32(&S->nu_full), 2 * kNuBytes + kKBytes);
        for (int s = 0; s < D / 64; ++s) {
          tma_load_2d(&himap, smem_u32(nuh + s * CP * 128), smem_u32(&S->nu_full), s * 64, h * CP);
          tma_load_2d(&lomap, smem_u32(nul + s * CP * 128), smem_u32(&S->nu_full), s * 64, h * CP);
        }
        bulk_load(smem_u32(kparts), kimg + static_cast<size_t>(h) * CP * kExtraK, kKBytes,
                  smem_u32(&S->nu_full));
        nu_pend = true;
        if (!mbar_wait(smem_u32(&S->nu_full), nu_par, abort)) return false;
        nu_pend = false;
        nu_par ^= 1u;
        return true;
      };
      // publish accumulator ii's tile (head -1: the end of the stream); the
      // scorers read the slot before they free accumulator ii - 2
      auto publish = [&](int ii, int h, int tt) -> bool {
        const int b = ii & 1;
        if (ii >= 2 && !mbar_wait(smem_u32(&S->t_free[b]), ((ii >> 1) - 1) & 1, abort)) return false;
        S->tile_h[b] = h;
        S->tile_t[b] = tt;
        mbar_arrive(smem_u32(&S->info_full[b]));
        return true;
      };
      const uint32_t ha = smem_u32(nuh), la = smem_u32(nul);
      const uint64_t ad_k = plain_desc(smem_u32(ones), 128, 256);
      const uint64_t bd_k = plain_desc(smem_u32(kparts), 128, 256);
#ifdef SVOO_TEST_STALL
      bool ok = mbar_wait(smem_u32(&S->stall), 0, abort);  // nothing completes it
#else
      bool ok = true;
#endif
      int loaded_h = -1;
      ok = ok && fetch(1);
      for (int ii = 0; ok && ii < min(known, 2); ++ii) ok = load_tile(ii);
      for (int ii = 0; ok; ++ii) {
        if (ii >= known) {  // the end of the stream
          publish(ii, -1, 0);
          break;
        }
        const int h = th[ii & 3], tt = tti[ii & 3], b = ii & 1;
        for (int s = 0; ok && s < kSpt; ++s) {
          const int q = ii * kSpt + s, slot = q % kStages;
          ok = mbar_wait(smem_u32(&S->xs_full[slot]), (q / kStages) & 1, abort);
          if (ok) xs_pend &= ~(1u << slot);
        }
        if (!ok || !publish(ii, h, tt)) break;  // also: accumulator b is free again
        if (h != loaded_h) {
          if (!load_nu(h)) break;
          loaded_h = h;
        }
        tc_fence_after();
        const uint32_t dt = tmem + b * CP;
        for (int s = 0; s < kSpt; ++s) {  // stage s: k chunks 4s .. 4s + 3 of the hi and lo products
          const int slot = (ii * kSpt + s) % kStages;
          const uint32_t xa = smem_u32(xs + slot * kStageBytes);
#pragma unroll
          for (int kq = 0; kq < 4; ++kq)
            umma_f16(dt, sw128_desc(xa + kq * 32, 16, 1024), sw128_desc(ha + s * CP * 128 + kq * 32, 16, 1024),
                     idesc, (s > 0 || kq > 0) ? 1u : 0u);
#pragma unroll
          for (int kq = 0; kq < 4; ++kq)
            umma_f16(dt, sw128_desc(xa + kq * 32, 16, 1024), sw128_desc(la + s * CP * 128 + kq * 32, 16, 1024),
                     idesc, 1u);
          umma_commit(smem_u32(&S->xs_free[slot]));  // the stage goes back once these are done
        }
        umma_f16(dt, ad_k, bd_k, idesc, 1u);
        umma_commit(smem_u32(&S->t_full[b]));
        mma_last = ii;
        // two tiles ahead
        ok = fetch(ii + 2);
        if (ok && ii + 2 < known) ok = load_tile(ii + 2);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ scorers
    const int lq = warp & 3;          // TMEM lane quarter
    const int cq = (warp - 1) >> 2;   // column quarter
    const int r = lq * 32 + lane;     // tile row
    const int quad_bar = 1 + lq;      // named barrier of the lane quarter's four warps
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(lq * 32) << 16);
    int cur_h = -1;
    float max_nrm = 0.f, max_kap = 0.f;
    for (int ii = 0;; ++ii) {
      const int b = ii & 1;
      const uint32_t ph = (ii >> 1) & 1;
      // the accumulator's tile, then (for a real tile) its MMA is complete
      bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->info_full[b]), ph, abort));
      const int h = ok ? S->tile_h[b] : -1;
      const int tt = ok ? S->tile_t[b] : 0;
      if (ok && h >= 0) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->t_full[b]), ph, abort));
      const bool done = !ok || h < 0;  // a timeout, or the end of the stream
      const int tok = tt * kTileRows + r;
      float xsq = 0.f;
      float v[kQCols];
      if (!done) {
        tc_fence_after();
        if (h != cur_h) {  // the head's bound maxima
          float mn = 0.f, mk = 0.f;
#pragma unroll
          for (int p = 0; p < CP / kNuCl; ++p) {
            const float2 m = __ldg(numax + h * (CP / kNuCl) + p);
            mn = fmaxf(mn, m.x);
            mk = fmaxf(mk, m.y);
          }
          max_nrm = mn;
          max_kap = mk;
          cur_h = h;
        }
        if (tok < nv) xsq = __ldg(xnorm + static_cast<size_t>(h) * nv + tok);
        // this quarter's scores into registers; then the accumulator is free
        const uint32_t ta = lane_base + b * CP + cq * kQCols;
        tmem_ld32f(ta, v);
        if constexpr (kLoads == 2) tmem_ld32f(ta + 32, v + 32);
        tmem_wait_ld_f(v);
        if constexpr (kLoads == 2) tmem_wait_ld_f(v + 32);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&S->t_free[b]));
        float m4[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
        for (int c = 4; c + 7 < kQCols + 4; c += 8) {
          m4[0] = fmax3(m4[0], v[c], v[c + 1]);
          m4[1] = fmax3(m4[1], v[c + 2], v[c + 3]);
          if (c + 4 < kQCols) {
            m4[2] = fmax3(m4[2], v[c + 4], v[c + 5]);
            m4[3] = fmax3(m4[3], v[c + 6], v[c + 7]);
          }
        }
        S->mq[cq][r] = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]);
      }
      // the four warps of the lane quarter leave together
      if (named_sync_or(quad_bar, 128, done ? 1 : 0)) break;
      // candidates of this quarter within 2E of the row maximum
      const float U = fmaxf(fmaxf(S->mq[0][r], S->mq[1][r]), fmaxf(S->mq[2][r], S->mq[3][r]));
      const float thr = U - ldexpf(sqrtf(xsq) * max_nrm + 0.5f * max_kap, -12);
      uint32_t mask[kLoads];
#pragma unroll
      for (int w32 = 0; w32 < kLoads; ++w32) {
        uint32_t p8[8];  // eight partial masks keep the OR chains short
#pragma unroll
        for (int u = 0; u < 8; ++u) p8[u] = 0u;
#pragma unroll
        for (int q = 0; q < 32; ++q) mark_ge(p8[q & 7], v[w32 * 32 + q], thr, 1u << q);
        mask[w32] = ((p8[0] | p8[1]) | (p8[2] | p8[3])) | ((p8[4] | p8[5]) | (p8[6] | p8[7]));
      }
      uint64_t mm = mask[0];
      if constexpr (kLoads == 2) mm |= static_cast<uint64_t>(mask[1]) << 32;
      const int k = __popcll(mm);
      reinterpret_cast<volatile uint8_t*>(&S->kc[r])[cq] = static_cast<uint8_t>(min(k, 255));
      named_sync(quad_bar, 128);
      // the row's decision, the same in the four warps
      const uint32_t kw = S->kc[r];
      const int k0 = kw & 255, k1 = (kw >> 8) & 255, k2 = (kw >> 16) & 255, k3 = kw >> 24;
      const int total = (k0 + k1) + (k2 + k3);
      const int kmax = max(max(k0, k1), max(k2, k3));
      const int before = cq == 0 ? 0 : cq == 1 ? k0 : cq == 2 ? k0 + k1 : (k0 + k1) + k2;
      const bool row = tok < nv;
      const bool listable = row && total >= 2 && total <= kDeferCand && kmax <= kQuarterCand;
      const long long grp = (static_cast<long long>(h) * ntiles + tt) * 4 + lq;
      DeferGroup* G = defer + grp;
      int32_t* arow = assign + static_cast<size_t>(h) * nv + tok;
      bool minus2 = false;
      if (row && total == 1) {
        if (k == 1) {  // the single candidate is this quarter's
          const int j = cq * kQCols + (__ffsll(static_cast<long long>(mm)) - 1);
          minus2 = j >= C;  // a padding column (only with non-finite input)
          *arow = minus2 ? -2 : j;
        }
      } else if (listable) {
#pragma unroll 1
        for (int u = 0; u < k; ++u) {
          const int q = __ffsll(static_cast<long long>(mm)) - 1;
          mm &= mm - 1;
          G->cand[lane][before + u] = static_cast<uint8_t>(cq * kQCols + q);
        }
      } else if (row && cq == 0) {  // too many candidates, or none: every cluster
        minus2 = true;
        *arow = -2;
      }
      if (cq == 0) G->n[lane] = static_cast<uint8_t>(listable ? total : 0);
      const unsigned dm = __ballot_sync(0xffffffffu, listable);
      const unsigned any2 = __ballot_sync(0xffffffffu, minus2);
      // word cq of the group: the listed rows (word 0) and kDeferAll
      if (lane == 0) defer_count[grp * 4 + cq] = (cq == 0 ? __popc(dm) : 0) | (any2 ? kDeferAll : 0);
    }
  }
  __syncthreads();
  if (*abort && tid == 0) {
    report_error(err, kErrTimeoutCluster);
    // copies and MMAs still in flight complete before the buffers go away
    for (int slot = 0; slot < kStages; ++slot)
      if (xs_pend & (1u << slot)) mbar_wait_cleanup(smem_u32(&S->xs_full[slot]), xs_par[slot]);
    if (nu_pend) mbar_wait_cleanup(smem_u32(&S->nu_full), nu_par);
    if (mma_last >= 0) mbar_wait_cleanup(smem_u32(&S->t_full[mma_last & 1]), (mma_last >> 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 2 * CP);
}

// ---------------------------------------------------------------- fixup
//
// Decides the rows the scorers could not, exactly: score kappa_j - 2 x.nu_j
// in fp64 over the whole bf16 row (the row is re-read in 16-byte pieces per
// cluster; they hit L1 and keep the register count low).
template <int D>
__device__ __forceinline__ double exact_score(const uint16_t* __restrict__ xrow, const double* __restrict__ nj,
                                              double kap_j) {
  // eight independent fp64 FMA chains, summed pairwise: an fp64 FMA's
  // dependent latency is long on this GPU, so short chains matter; eight
  // (not sixteen) leave registers for 12 blocks of fixup_kernel per SM, which
  // measured faster
  double e[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) e[u] = 0.0;
#pragma unroll 2
  for (int i = 0; i < D; i += 16) {
    const uint4 xa = __ldg(reinterpret_cast<const uint4*>(xrow + i));
    const uint4 xb = __ldg(reinterpret_cast<const uint4*>(xrow + i + 8));
    const uint32_t w[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const double2 nv = __ldg(reinterpret_cast<const double2*>(nj + i + 2 * u));
      e[u] = fma(static_cast<double>(__uint_as_float(w[u] << 16)), nv.x, e[u]);
      e[u] = fma(static_cast<double>(__uint_as_float(w[u] & 0xffff0000u)), nv.y, e[u]);
    }
  }
#pragma unroll
  for (int step = 4; step > 0; step >>= 1)
#pragma unroll
    for (int u = 0; u < step; ++u) e[u] += e[u + step];
  return kap_j - 2.0 * e[0];
}

// The label of a row against every cluster (rows whose candidates were not
// listed): each lane scores its clusters j = lane, lane + 32, ... exactly,
// kappa_j - 2 x.nu_j in fp64 over the whole row, then the warp takes the
// minimum, ties to the smaller j.
template <int D>
__device__ int decide_all(const uint16_t* __restrict__ xrow, const double* __restrict__ nu64h,
                          const double* __restrict__ kap, int C, int lane) {
  double best = INFINITY;
  int bj = 0x7fffffff;
  for (int j = lane; j < C; j += 32) {
    const double sc = exact_score<D>(xrow, nu64h + static_cast<size_t>(j) * D, kap[j]);
    if (sc < best) {  // j ascends within a lane
      best = sc;
      bj = j;
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    const double ob = __shfl_xor_sync(0xffffffffu, best, o);
    const int oj = __shfl_xor_sync(0xffffffffu, bj, o);
    if (ob < best || (ob == best && oj < bj)) {
      best = ob;
      bj = oj;
    }
  }
  return bj;
}

// grid: ceil(groups / kFixWarps) blocks of kFixWarps warps, groups = B*H *
// tiles * 4: one warp per 32-row group. Listed rows: the group's (row,
// candidate) pairs are laid out row after row, 32 per round, and each lane
// scores one pair exactly, kappa_j - 2 x.nu_j in fp64; a segmented minimum
// over the lanes of each row's run (ties to the smaller j) goes to the row's
// own lane, which keeps the row's best over the rounds. Rows labelled -2 (by
// the scorers, or here for a list that does not look right): the whole warp
// compares every cluster (decide_all). 12 blocks per SM: more warps in flight
// hide the fp64 latency better than spill-free registers did.
constexpr int kFixWarps = 4;

__device__ __forceinline__ bool better(double sa, int ja, double sb, int jb) {
  return sa < sb || (sa == sb && ja < jb);  // NaN never wins
}

template <int D, int CP>
__global__ void __launch_bounds__(kFixWarps * 32, 12)
    fixup_kernel(const uint16_t* __restrict__ x, int N, int nv, int C, int BH, int ntiles,
                 const double* __restrict__ nu64, const double* __restrict__ kappa64,
                 int32_t* __restrict__ assign, const int32_t* __restrict__ defer_count,
                 const DeferGroup* __restrict__ defer, int* __restrict__ err) {
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  if (timed_out_before(err)) return;  // the scorers may not have written their lists
  const long long ngrp = static_cast<long long>(BH) * ntiles * 4;
  const long long g = static_cast<long long>(blockIdx.x) * kFixWarps + wi;
  if (g >= ngrp) return;  // warp-uniform
  const int4 dc = *reinterpret_cast<const int4*>(defer_count + g * 4);
  bool any_all = ((dc.x | dc.y | dc.z | dc.w) & kDeferAll) != 0;
  const int h = static_cast<int>(g / (static_cast<long long>(ntiles) * 4));
  const int r4 = static_cast<int>(g - static_cast<long long>(h) * ntiles * 4);
  const int row0 = (r4 >> 2) * kTileRows + (r4 & 3) * 32;  // the group's first token
  int32_t* asg = assign + static_cast<size_t>(h) * nv;
  const double* nuh = nu64 + static_cast<size_t>(h) * C * D;
  const double* kap = kappa64 + static_cast<size_t>(h) * CP;
  if ((dc.x & (kDeferAll - 1)) > 0) {
    const DeferGroup* G = defer + g;
    const int tok = row0 + lane;
    int n = G->n[lane];
    if (n > kDeferCand || tok >= nv) n = 0;  // not listed (or not a record to trust)
    int off = n;  // inclusive prefix sum of the counts over the rows
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, off, o);
      if (lane >= o) off += t;
    }
    const int total = __shfl_sync(0xffffffffu, off, 31);
    off -= n;  // exclusive: row l's pairs are off_l .. off_l + n_l - 1
    double best = INFINITY;  // this lane's row, over the rounds
    int bj = 0x7fffffff;
    bool bad = false;
    // every lane runs every round (the shuffles need the whole warp)
    for (int base = 0; base < total; base += 32) {
      const int it = base + lane;
      int s = 0;  // the row of pair it: the last row l with off_l <= it (rows
                  // without pairs share the next row's offset, so they are passed over)
#pragma unroll
      for (int step = 16; step > 0; step >>= 1) {
        const int off_c = __shfl_sync(0xffffffffu, off, s + step);
        if (off_c <= it) s += step;
      }
      const int off_s = __shfl_sync(0xffffffffu, off, s);
      double sc = NAN;
      int j = 0x7fffffff;
      if (it < total) {
        j = G->cand[s][it - off_s];
        if (j < C)
          sc = exact_score<D>(x + (static_cast<size_t>(h) * N + row0 + s) * D, nuh + static_cast<size_t>(j) * D,
                              kap[j]);
        else
          j = -1;  // a candidate that does not look right
      }
      // segmented minimum: a row's pairs are a run of consecutive lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const double sc2 = __shfl_down_sync(0xffffffffu, sc, o);
        const int j2 = __shfl_down_sync(0xffffffffu, j, o);
        const int s2 = __shfl_down_sync(0xffffffffu, s, o);
        const int it2 = it + o;
        if (lane + o < 32 && it2 < total && s2 == s) {
          if (j2 < 0 || j < 0) j = -1;  // a bad candidate anywhere in the row's run
          else if (better(sc2, j2, sc, j)) {
            sc = sc2;
            j = j2;
          }
        }
      }
      // the run of row `lane` in this round starts at lane max(off - base, 0)
      const bool mine = n > 0 && off < base + 32 && off + n > base;
      const int head = max(off - base, 0);
      const double rs = __shfl_sync(0xffffffffu, sc, mine ? head : lane);
      const int rj = __shfl_sync(0xffffffffu, j, mine ? head : lane);
      if (mine) {
        if (rj < 0) bad = true;
        else if (better(rs, rj, best, bj)) {
          best = rs;
          bj = rj;
        }
      }
    }
    if (n > 0) {
      const int lbl = (!bad && bj < C) ? bj : -2;  // a candidate that does not look right: every cluster
      asg[tok] = lbl;
      any_all = any_all || lbl == -2;
    }
    any_all = __any_sync(0xffffffffu, any_all);
  }
  if (!any_all) return;
  // rows labelled -2: every cluster, the whole warp per row
  __syncwarp();
  const int tok = row0 + lane;
  unsigned all = __ballot_sync(0xffffffffu, tok < nv && asg[tok] == -2);
  while (all) {
    const int l = __ffs(all) - 1;
    all &= all - 1;
    const int lbl = decide_all<D>(x + (static_cast<size_t>(h) * N + row0 + l) * D, nuh, kap, C, lane);
    if (lane == 0) asg[row0 + l] = lbl;
  }
}

// ---------------------------------------------------------------- update
//
// Member sums are exact: components with |x| < 2^-24 count as zero, so every
// partial sum is a multiple of 2^-31 below 2^22 in magnitude and fp64 holds it
// exactly; the order of the additions (and of the fp64 atomic additions of
// partial sums) changes nothing, and the centroid fp32(sum / n) is the one the
// exact mean rounds to.

constexpr int kMaxClusters = 256;
constexpr int kUpdTokens = 2048;     // consecutive tokens per CTA
constexpr int kUpdThreads = 256;
constexpr int kUpdWarps = kUpdThreads / 32;

// A bf16 value, given as the fp32 bit pattern b (the bf16 in the upper half),
// to fp64 with |x| < 2^-24 counted as zero.
__device__ __forceinline__ double bf16_to_f64_flushed(uint32_t b) {
  const float v = __uint_as_float(b);
  return fabsf(v) < 5.9604644775390625e-08f ? 0.0 : static_cast<double>(v);  // 2^-24
}

__device__ __forceinline__ void red_f64(double* dst, double v) {
  asm volatile("red.global.add.f64 [%0], %1;" ::"l"(dst), "d"(v) : "memory");
}

__device__ __forceinline__ void red_s32(int32_t* dst, int v) {
  asm volatile("red.global.add.s32 [%0], %1;" ::"l"(dst), "r"(v) : "memory");
}

// grid (ceil(nv / kUpdTokens), BH), block kUpdThreads, one chunk of
// kUpdTokens consecutive tokens per CTA. prev == nullptr: every token is an
// entry +x for its label. Otherwise (the incremental update of a whole call:
// the side's sums and counts of its previous half-step are kept) only the
// tokens whose label changed since prev are entries, +x for the new label and
// -x for the old one, and prev is brought up to date; every partial sum is
// then a sum of the same exact fp64 contributions as a full pass, so the
// result has the same bits. The CTA groups its entries by cluster in shared
// memory (the order inside a cluster is irrelevant: the sums are exact), adds
// each cluster's count change to counts[h][j], and each warp sums a
// contiguous run of the grouped order in fp64, adding every cluster's
// partial sum to sums[h][j] once. The rows it reads lie in the chunk's slice
// of X.
template <int D>
__global__ void __launch_bounds__(kUpdThreads)
    update_kernel(const uint16_t* __restrict__ x, int N, int nv, int C, const int32_t* __restrict__ assign,
                  int32_t* __restrict__ prev, double* __restrict__ sums, int32_t* __restrict__ counts,
                  int* __restrict__ err) {
  constexpr int kPer = D / 32;
  constexpr int kBatch = 16;
  constexpr uint16_t kNeg = 0x8000;  // entry flag: subtract the row
  __shared__ int cnt[kMaxClusters];   // entries per cluster
  __shared__ int dlt[kMaxClusters];   // count change per cluster
  __shared__ int base[kMaxClusters + 1];
  __shared__ uint16_t order[2 * kUpdTokens];
  __shared__ uint16_t moved[kUpdTokens];  // incremental: the chunk's tokens whose label changed
  __shared__ int n_moved;
  const int h = blockIdx.y, c0 = blockIdx.x * kUpdTokens;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (timed_out_before(err)) return;  // labels of an aborted step are not to be trusted
  const int n = min(kUpdTokens, nv - c0);
  const int32_t* a = assign + static_cast<size_t>(h) * nv + c0;
  int32_t* pv = prev ? prev + static_cast<size_t>(h) * nv + c0 : nullptr;
  for (int j = tid; j < C; j += kUpdThreads) cnt[j] = dlt[j] = 0;
  if (tid == 0) n_moved = 0;
  __syncthreads();
  // incremental: list the moved tokens first (most did not move), so the two
  // grouping passes below run over them only
  if (pv) {
    for (int t0 = warp * 32; t0 < n; t0 += kUpdThreads) {
      const int t = t0 + lane;
      const bool mv = t < n && a[t] != pv[t];
      const unsigned bm = __ballot_sync(0xffffffffu, mv);
      int at = 0;
      if (lane == 0 && bm) at = atomicAdd(&n_moved, __popc(bm));
      at = __shfl_sync(0xffffffffu, at, 0);
      if (mv) moved[at + __popc(bm & ((1u << lane) - 1u))] = static_cast<uint16_t>(t);
    }
    __syncthreads();
  }
  const int n_items = pv ? n_moved : n;  // tokens the grouping passes visit
  auto token_of = [&](int i) { return pv ? (i < n_items ? static_cast<int>(moved[i]) : n) : i; };
  // a token's entries: (l, +) and, when it moved, (o, -); -1 for none (and
  // for t = n, past the chunk)
  auto entries = [&](int t, int& l, int& o) {
    l = t < n ? a[t] : -1;
    o = -1;
    if (t < n && (l < 0 || l >= C)) {
      report_error(err, kErrBadLabel);
      l = -1;
    }
    if (pv && t < n) {
      const int old = pv[t];
      if (old == l) {
        l = -1;  // unchanged: no entry
      } else if (old >= 0 && old < C) {
        o = old;
      } else if (l >= 0) {
        report_error(err, kErrBadLabel);
        l = -1;
      }
    }
  };
  // labels come in runs (neighbouring tokens share clusters): lanes with equal
  // labels add to the shared counters once, through their lowest lane
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = warp * 32; i0 < n_items; i0 += kUpdThreads) {
    int l, o;
    entries(token_of(i0 + lane), l, o);
    const unsigned pl = __match_any_sync(0xffffffffu, l);
    if (l >= 0 && (pl & lt) == 0) {
      atomicAdd(&cnt[l], __popc(pl));
      atomicAdd(&dlt[l], __popc(pl));
    }
    if (pv) {
      const unsigned po = __match_any_sync(0xffffffffu, o);
      if (o >= 0 && (po & lt) == 0) {
        atomicAdd(&cnt[o], __popc(po));
        atomicAdd(&dlt[o], -__popc(po));
      }
    }
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the entry counts
    int run = 0;
    for (int j0 = 0; j0 < C; j0 += 32) {
      const int j = j0 + lane;
      const int c = j < C ? cnt[j] : 0;
      int incl = c;
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (j < C) base[j] = run + incl - c;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) base[C] = run;
  }
  __syncthreads();
  for (int j = tid; j < C; j += kUpdThreads) {
    if (dlt[j] != 0) red_s32(&counts[static_cast<size_t>(h) * C + j], dlt[j]);
    cnt[j] = 0;
  }
  __syncthreads();
  for (int i0 = warp * 32; i0 < n_items; i0 += kUpdThreads) {
    const int t = token_of(i0 + lane);
    int l, o;
    entries(t, l, o);
    const unsigned pl = __match_any_sync(0xffffffffu, l);
    const int ll = __ffs(pl) - 1;
    int pos = 0;
    if (l >= 0 && lane == ll) pos = atomicAdd(&cnt[l], __popc(pl));
    pos = __shfl_sync(0xffffffffu, pos, ll);
    if (l >= 0) order[base[l] + pos + __popc(pl & lt)] = static_cast<uint16_t>(t);
    if (pv) {
      const unsigned po = __match_any_sync(0xffffffffu, o);
      const int lo = __ffs(po) - 1;
      int pos2 = 0;
      if (o >= 0 && lane == lo) pos2 = atomicAdd(&cnt[o], __popc(po));
      pos2 = __shfl_sync(0xffffffffu, pos2, lo);
      if (o >= 0) {
        order[base[o] + pos2 + __popc(po & lt)] = static_cast<uint16_t>(t | kNeg);
        pv[t] = a[t];  // the token's entries are placed: prev catches up
      }
    }
  }
  __syncthreads();
  const int nvalid = base[C];
  const int p0 = warp * nvalid / kUpdWarps, p1 = (warp + 1) * nvalid / kUpdWarps;
  if (p0 >= p1) return;
  // the cluster of position p0: the last j with base[j] <= p0
  int lo_j = 0, hi_j = C - 1;
  while (lo_j < hi_j) {
    const int mid = (lo_j + hi_j + 1) >> 1;
    if (base[mid] <= p0) lo_j = mid;
    else hi_j = mid - 1;
  }
  int j = lo_j, end = base[j + 1];
  const uint16_t* xc = x + (static_cast<size_t>(h) * N + c0) * D;
  double acc[2][kPer];  // even and odd entries of a batch: two short dependency chains
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[0][u] = acc[1][u] = 0.0;
  bool any = false;
  auto flush = [&]() {
    if (any) {
      double* dst = sums + (static_cast<size_t>(h) * C + j) * D + kPer * lane;
#pragma unroll
      for (int u = 0; u < kPer; ++u) red_f64(dst + u, acc[0][u] + acc[1][u]);
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) acc[0][u] = acc[1][u] = 0.0;
    any = false;
  };
  for (int pb = p0; pb < p1; pb += kBatch) {
    uint32_t w0[kBatch], w1[kBatch];
    uint32_t neg = 0u;  // bit q: entry q subtracts its row
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {  // the batch's rows in flight together
      w0[q] = 0u;
      w1[q] = 0u;
      if (pb + q < p1) {
        const uint16_t e = order[pb + q];
        const int t = e & (kNeg - 1);
        neg |= (e & kNeg) ? (1u << q) : 0u;
        if (kPer == 4) {
          const uint2 v = __ldg(reinterpret_cast<const uint2*>(xc + static_cast<size_t>(t) * D) + lane);
          w0[q] = v.x;
          w1[q] = v.y;
        } else {
          w0[q] = __ldg(reinterpret_cast<const uint32_t*>(xc + static_cast<size_t>(t) * D) + lane);
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int p = pb + q;
      if (p >= p1) break;
      while (p >= end && j + 1 < C) {  // next non-empty cluster
        flush();
        ++j;
        end = base[j + 1];
      }
      // +-1 times an exact value is exact
      const double sg = ((neg >> q) & 1u) ? -1.0 : 1.0;
      acc[q & 1][0] = fma(sg, bf16_to_f64_flushed(w0[q] << 16), acc[q & 1][0]);
      acc[q & 1][1] = fma(sg, bf16_to_f64_flushed(w0[q] & 0xffff0000u), acc[q & 1][1]);
      if (kPer == 4) {
        acc[q & 1][2] = fma(sg, bf16_to_f64_flushed(w1[q] << 16), acc[q & 1][2]);
        acc[q & 1][3] = fma(sg, bf16_to_f64_flushed(w1[q] & 0xffff0000u), acc[q & 1][3]);
      }
      any = true;
    }
  }
  flush();
}

// centroid = fp32(sum / n) where n > 0 (an empty cluster keeps its centroid),
// sizes = n; resets the chunk counters and, unless `keep` (the call's
// incremental sums), the sums and counts.
__global__ void finalize_kernel(double* __restrict__ sums, int32_t* __restrict__ counts,
                                float* __restrict__ cent, int32_t* __restrict__ sizes,
                                int32_t* __restrict__ head_next, int C, int d, int keep) {
  const int h = blockIdx.y, j = blockIdx.x, i = threadIdx.x;
  const int n = counts[h * C + j];
  const size_t e = (static_cast<size_t>(h) * C + j) * d + i;
  if (n > 0) cent[e] = static_cast<float>(sums[e] / static_cast<double>(n));
  if (!keep) sums[e] = 0.0;
  __syncthreads();
  if (i == 0) {
    sizes[h * C + j] = n;
    if (!keep) counts[h * C + j] = 0;
  }
  if (i == 0 && j == 0) head_next[h] = 0;
}

// ---------------------------------------------------------------- host side

namespace {

struct StepWs {
  double* M;
  double* nu64;
  uint16_t* nu_hi;
  uint16_t* nu_lo;
  double* kappa64;
  uint16_t* kimg;
  float2* numax;
  double* sums;
  int32_t* counts;
  int32_t* head_next;
  float* xnorm;
  int32_t* defer_count;
  DeferGroup* defer;
};

// columns of the scoring MMA: the cluster count padded so that four threads
// per row read one or two 32-column TMEM chunks each
inline int score_cols(int c) { return c <= 128 ? 128 : 256; }

size_t carve_step(void* ws, int BH, int d, int Cmax, int nv, StepWs* out) {
  Carver cv(ws);
  const int CP = score_cols(Cmax);
  const size_t ntiles = (static_cast<size_t>(nv) + kTileRows - 1) / kTileRows;
  StepWs w;
  w.M = cv.take<double>(static_cast<size_t>(BH) * d * d);
  w.nu64 = cv.take<double>(static_cast<size_t>(BH) * Cmax * d);
  w.nu_hi = cv.take<uint16_t>(static_cast<size_t>(BH) * CP * d);
  w.nu_lo = cv.take<uint16_t>(static_cast<size_t>(BH) * CP * d);
  w.kappa64 = cv.take<double>(static_cast<size_t>(BH) * CP);
  w.kimg = cv.take<uint16_t>(static_cast<size_t>(BH) * CP * kExtraK);
  w.numax = cv.take<float2>(static_cast<size_t>(BH) * (CP / kNuCl));
  w.sums = cv.take<double>(static_cast<size_t>(BH) * Cmax * d);
  w.counts = cv.take<int32_t>(static_cast<size_t>(BH) * Cmax);
  w.head_next = cv.take<int32_t>(static_cast<size_t>(BH));
  w.xnorm = cv.take<float>(static_cast<size_t>(BH) * nv);
  w.defer_count = cv.take<int32_t>(static_cast<size_t>(BH) * ntiles * 4 * 4);
  w.defer = cv.take<DeferGroup>(static_cast<size_t>(BH) * ntiles * 4);
  if (out) *out = w;
  return cv.used + 256;
}

// The member sums of one side of a whole svoo_cluster call, kept from one
// half-step of that side to the next, with the labels they were summed for.
struct SideSums {
  double* sums;
  int32_t* counts;
  int32_t* prev;
};
// kUpdFull: sums from scratch into the step's scratch, cleared afterwards (a
// lone half-step); kUpdFullKeep: from scratch into the side's kept sums (its
// first half-step of a call); kUpdIncr: only the changed labels move.
constexpr int kUpdFull = 0, kUpdFullKeep = 1, kUpdIncr = 2;

template <int D, int CP>
svoo_status launch_assign(const CUtensorMap& xmap, const svoo_shape* sh, const void* x, int C,
                          const StepWs& w, int32_t* assign, const float* xnorm, double* sums,
                          int32_t* counts, int32_t* prev, int upd, int32_t* dev_err, cudaStream_t st) {
  const int BH = bh_of(sh), N = sh->N, nv = nvideo_of(sh);
  const size_t smem = 1024 + kAssignHeader + static_cast<size_t>(kStages) * kStageBytes +
                      2 * static_cast<size_t>(CP) * D * 2 + (kTileRows + CP) * kExtraK * 2;
  if (cudaFuncSetAttribute(assign_kernel<D, CP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SVOO_ERR_CUDA;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return SVOO_ERR_CUDA;
  const int ntiles = (nv + kTileRows - 1) / kTileRows;
  const long long chunks = static_cast<long long>(BH) * ((ntiles + kChunkTiles - 1) / kChunkTiles);
  const int grid = static_cast<int>(chunks < sms ? chunks : sms);
  CUtensorMap himap, lomap;
  if (encode_tiled_2d(&himap, w.nu_hi, static_cast<uint64_t>(BH) * CP, D, CP, 64) != CUDA_SUCCESS ||
      encode_tiled_2d(&lomap, w.nu_lo, static_cast<uint64_t>(BH) * CP, D, CP, 64) != CUDA_SUCCESS)
    return SVOO_ERR_CUDA;
  assign_kernel<D, CP><<<grid, kAssignThreads, smem, st>>>(
      xmap, himap, lomap, N, nv, C, BH, w.kimg, w.numax, w.head_next, assign, w.defer_count, w.defer,
      xnorm, dev_err);
  if (cudaGetLastError() != cudaSuccess) return SVOO_ERR_CUDA;
  const long long groups = static_cast<long long>(BH) * ntiles * 4;
  fixup_kernel<D, CP><<<static_cast<unsigned>((groups + kFixWarps - 1) / kFixWarps), kFixWarps * 32, 0, st>>>(
      static_cast<const uint16_t*>(x), N, nv, C, BH, ntiles, w.nu64, w.kappa64, assign, w.defer_count,
      w.defer, dev_err);
  if (cudaGetLastError() != cudaSuccess) return SVOO_ERR_CUDA;
  update_kernel<D><<<dim3((nv + kUpdTokens - 1) / kUpdTokens, BH), kUpdThreads, 0, st>>>(
      static_cast<const uint16_t*>(x), N, nv, C, assign, upd == kUpdIncr ? prev : nullptr, sums, counts,
      dev_err);
  if (upd == kUpdFullKeep &&
      cudaMemcpyAsync(prev, assign, sizeof(int32_t) * BH * static_cast<size_t>(nv), cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return SVOO_ERR_CUDA;
  return SVOO_OK;
}

// |x|^2 of the video tokens of x into xn (fp32 [BH][nv]).
svoo_status launch_xnorm(const svoo_shape* sh, const void* x, float* xn, cudaStream_t st) {
  const int BH = bh_of(sh), nv = nvideo_of(sh);
  const dim3 grid((nv + 31) / 32, BH);
  if (sh->d == 128)
    xnorm_kernel<128><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), sh->N, nv, xn);
  else
    xnorm_kernel<64><<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(x), sh->N, nv, xn);
  return cudaGetLastError() == cudaSuccess ? SVOO_OK : SVOO_ERR_CUDA;
}

// One half-step. metric_cent == nullptr: identity metric. xnorm: |x|^2 of
// this side's tokens, already computed for the whole call; without it the
// step computes it into its own scratch. side (with upd kUpdFullKeep /
// kUpdIncr): the side's kept sums of a whole call; without it, the step's own
// scratch.
svoo_status run_step(const svoo_shape* sh, const void* x, int C, float* cent, int32_t* sizes,
                     int32_t* assign, const float* metric_cent, const int32_t* metric_sizes,
                     int metric_C, const StepWs& w, int32_t* dev_err, cudaStream_t st,
                     int zero_C, const float* xnorm = nullptr, const SideSums* side = nullptr,
                     int upd = kUpdFull) {
  double* sums = side ? side->sums : w.sums;
  int32_t* counts = side ? side->counts : w.counts;
  int32_t* prev = side ? side->prev : nullptr;
  if (!side) upd = kUpdFull;
  const int BH = bh_of(sh), d = sh->d, N = sh->N;
  const int CP = score_cols(C);
  // finalize_kernel re-zeroes what a step used, so only the first step of a
  // call clears the sums and the chunk counters (for the call's largest
  // cluster count).
  if (zero_C > 0) {
    if (cudaMemsetAsync(w.sums, 0, sizeof(double) * BH * static_cast<size_t>(zero_C) * d, st) != cudaSuccess ||
        cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * BH * static_cast<size_t>(zero_C), st) != cudaSuccess ||
        cudaMemsetAsync(w.head_next, 0, sizeof(int32_t) * BH, st) != cudaSuccess)
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
  metric_nu_kernel<<<dim3(CP / kNuCl, BH), 128, metric_nu_smem(d), st>>>(
      metric_cent ? w.M : nullptr, cent, C, CP, d, w.nu64, w.nu_hi, w.nu_lo, w.kappa64, w.kimg,
      w.numax);
  CUtensorMap xmap;
  if (encode_tiled_2d(&xmap, x, static_cast<uint64_t>(BH) * N, d, kTileRows, 64) != CUDA_SUCCESS)
    return SVOO_ERR_CUDA;
  if (!xnorm) {  // a lone half-step
    if (launch_xnorm(sh, x, w.xnorm, st) != SVOO_OK) return SVOO_ERR_CUDA;
    xnorm = w.xnorm;
  }
  svoo_status s;
  if (d == 128)
    s = CP == 256 ? launch_assign<128, 256>(xmap, sh, x, C, w, assign, xnorm, sums, counts, prev, upd, dev_err, st)
                  : launch_assign<128, 128>(xmap, sh, x, C, w, assign, xnorm, sums, counts, prev, upd, dev_err, st);
  else
    s = CP == 256 ? launch_assign<64, 256>(xmap, sh, x, C, w, assign, xnorm, sums, counts, prev, upd, dev_err, st)
                  : launch_assign<64, 128>(xmap, sh, x, C, w, assign, xnorm, sums, counts, prev, upd, dev_err, st);
  if (s != SVOO_OK) return s;
  finalize_kernel<<<dim3(C, BH), d, 0, st>>>(sums, counts, cent, sizes, w.head_next, C, d,
                                             upd != kUpdFull ? 1 : 0);
  return launch_status();
}

bool cluster_counts_ok(int C) { return C >= 1 && C <= 256; }

// Workspace of a whole svoo_cluster call: one half-step's scratch, then per
// side (queries, keys) the per-token |x|^2 (fp32 [BH][N - n_text]) and the
// kept member sums (fp64 [BH][C][d]), counts and labels of its last half-step.
size_t carve_call(void* ws, const svoo_shape* sh, int n_qc, int n_kc, StepWs* w, float** xn_q, float** xn_k,
                  SideSums* sq, SideSums* sk) {
  const int Cmax = n_qc > n_kc ? n_qc : n_kc;
  const size_t step = carve_step(ws, bh_of(sh), sh->d, Cmax, nvideo_of(sh), w);
  Carver cv(ws ? static_cast<char*>(ws) + step : nullptr);
  const size_t BH = static_cast<size_t>(bh_of(sh));
  const size_t n = BH * nvideo_of(sh);
  float* a = cv.take<float>(n);
  float* b = cv.take<float>(n);
  if (xn_q) *xn_q = a;
  if (xn_k) *xn_k = b;
  SideSums q, k;
  q.sums = cv.take<double>(BH * n_qc * sh->d);
  q.counts = cv.take<int32_t>(BH * n_qc);
  q.prev = cv.take<int32_t>(n);
  k.sums = cv.take<double>(BH * n_kc * sh->d);
  k.counts = cv.take<int32_t>(BH * n_kc);
  k.prev = cv.take<int32_t>(n);
  if (sq) *sq = q;
  if (sk) *sk = k;
  return step + cv.used + 256;
}

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
  return carve_call(nullptr, shape, n_qc, n_kc, nullptr, nullptr, nullptr, nullptr, nullptr);
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
  size_t need = carve_step(workspace, BH, shape->d, step_clusters(C, metric_cent, metric_C), nvideo_of(shape), &w);
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
  float *xn_q = nullptr, *xn_k = nullptr;
  SideSums sq, sk;
  size_t need = carve_call(workspace, shape, n_qc, n_kc, &w, &xn_q, &xn_k, &sq, &sk);
  if (workspace_bytes < need) return SVOO_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // each side's kept sums start empty; its first half-step sums every member
  if (cudaMemsetAsync(sq.sums, 0, sizeof(double) * BH * static_cast<size_t>(n_qc) * d, st) != cudaSuccess ||
      cudaMemsetAsync(sq.counts, 0, sizeof(int32_t) * BH * static_cast<size_t>(n_qc), st) != cudaSuccess ||
      cudaMemsetAsync(sk.sums, 0, sizeof(double) * BH * static_cast<size_t>(n_kc) * d, st) != cudaSuccess ||
      cudaMemsetAsync(sk.counts, 0, sizeof(int32_t) * BH * static_cast<size_t>(n_kc), st) != cudaSuccess)
    return SVOO_ERR_CUDA;
  if (!warm) {
    init_centroids_kernel<<<dim3(n_qc, BH), d, 0, st>>>(static_cast<const uint16_t*>(q), N, nv, d, n_qc, q_cent);
    init_centroids_kernel<<<dim3(n_kc, BH), d, 0, st>>>(static_cast<const uint16_t*>(k), N, nv, d, n_kc, k_cent);
  }
  const int Cmax = n_qc > n_kc ? n_qc : n_kc;
  // |x|^2 of both sides' tokens (the inputs do not change during the call)
  if (launch_xnorm(shape, q, xn_q, st) != SVOO_OK || launch_xnorm(shape, k, xn_k, st) != SVOO_OK)
    return SVOO_ERR_CUDA;
  for (int it = 0; it < iters; ++it) {
    const bool ident = identity || (it == 0 && !warm);
    const int upd = it == 0 ? kUpdFullKeep : kUpdIncr;
    svoo_status s = run_step(shape, q, n_qc, q_cent, q_sizes, q_assign, ident ? nullptr : k_cent,
                             k_sizes, n_kc, w, dev_err, st, it == 0 ? Cmax : 0, xn_q, &sq, upd);
    if (s != SVOO_OK) return s;
    s = run_step(shape, k, n_kc, k_cent, k_sizes, k_assign, identity ? nullptr : q_cent, q_sizes,
                 n_qc, w, dev_err, st, 0, xn_k, &sk, upd);
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
  if (carve_step(nullptr, BH, shape->d, Cmax, nvideo_of(shape), nullptr) > kStaticScratchBytes)
    return SVOO_ERR_WORKSPACE;  // shape needs more than the fixed scratch holds
  int dev = 0;
  void* base = scratch_address(&dev);
  if (!base) return SVOO_ERR_CUDA;
  StepWs w;
  carve_step(base, BH, shape->d, Cmax, nvideo_of(shape), &w);
  return run_step(shape, x, C, cent, sizes, assign, metric_cent, metric_sizes, metric_C, w, dev_err,
                  static_cast<cudaStream_t>(stream), C);
}
