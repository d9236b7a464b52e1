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
//   assign_kernel     persistent, warp-specialised, dynamically scheduled:
//                     tcgen05 MMAs of 128-token tiles against [nu_hi | nu_lo]
//                     into double-buffered TMEM; per token the score
//                     kappa_j - 2 x.nu_j is bounded by the MMA error and a
//                     token with a single candidate takes it
//   fixup_kernel      the other tokens: candidates re-scored closer, then in
//                     fp64 (ties to the smaller j)
//   update_kernel     member sums in fp64, exact (so order-independent), per
//                     chunk of consecutive tokens grouped by label
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

// ---------------------------------------------------------------- assign
//
// Persistent, warp-specialised kernel, one CTA per SM. The (head, 128-token
// tile) space is handed out in chunks of kChunkTiles tiles of one head through
// per-head counters: a CTA starts at its own head and moves on to the next
// head with chunks left, so SMs that run this kernel faster take more chunks
// (on B200 some SMs ran the same tiles up to 1.5x slower than others, so a
// static split left the fast ones idle). Tile i of a CTA uses X buffer i % 2
// in shared memory and TMEM accumulator i % 2 (CP fp32 columns).
//   producer (warp 0)   TMA of the X tile, then one tcgen05 chain per tile:
//                       u = X . nu_hi^T + X . nu_lo^T + 1 . (-kappa/2)^T, the
//                       last term a 16-wide K chunk of ones against -kappa_j/2
//                       split into three bf16 parts, so u_j = x.nu_j - kappa_j/2
//                       and the score is kappa_j - 2 x.nu_j = -2 u_j.
//   scorers (warps 1-16) warp w reads TMEM lane quarter w % 4 (32 rows) and
//                       column quarter (w - 1) / 4: each thread loads its row's
//                       CP/4 scores into registers (then the accumulator goes
//                       back), the quarter's maximum; the four quarters of a
//                       row meet in shared memory for the row maximum U and
//                       the error bound E; then each thread lists its
//                       quarter's candidates u_j >= U - 2E (they contain the
//                       exact argmin of the score). The quarter-0 warp of a
//                       lane quarter decides its rows: one candidate is the
//                       label; several go to the tile's deferred list (up to
//                       kDeferSlots rows per 32 with up to kDeferCand
//                       candidates each, label -1) or, beyond that, get label
//                       -2 (all clusters); fixup_kernel decides them.
//
// Error bound: nu_hi + nu_lo equals nu to 2^-18 relative and the three kappa
// parts give kappa to 2^-26; the MMA's fp32 accumulation of 2d + 3 exact
// products adds at most (2d + 3) 2^-23 of the sum of their magnitudes, at most
// |x||nu_j| (1 + 2^-8) + |kappa_j| / 2. E = 2^-13 (|x| max|nu| + max|kappa| / 2)
// bounds |u_computed - u| with a factor of two to spare.

// |x|^2 of the tokens: computed by the scorers from the X tile (and, with
// kXnormStore, kept per token for the later half-steps of the same side), or
// loaded from that store (the inputs do not change between half-steps)
constexpr int kXnormCompute = 0, kXnormStore = 1, kXnormLoad = 2;

constexpr int kScorerWarps = 16;
constexpr int kAssignWarps = 1 + kScorerWarps;
constexpr int kAssignThreads = kAssignWarps * 32;
constexpr int kScorers = kScorerWarps * 32;
constexpr int kTileRows = 128;
constexpr int kQuarterCand = 4;      // candidates kept per column quarter
constexpr int kDeferSlots = 8;       // listed deferred rows per 32 rows of a tile
constexpr int kDeferCand = 8;        // candidates of a listed deferred row
constexpr int kDeferAll = 1 << 8;    // defer_count flag: some rows of the group have label -2
constexpr int kChunkTiles = 16;      // tiles per claimed chunk
constexpr int kAssignHeader = 12288; // AssignSmem, keeps the X buffers 1024-aligned
constexpr int kExtraK = 16;          // the kappa chunk of the MMA
// named barriers: 1..4 the four scorer warps of a TMEM lane quarter, 5 all scorers
constexpr int kBarScorers = 5;

// A row with several candidates, decided by fixup_kernel.
struct DeferRec {
  int32_t tok;
  int32_t n;                   // candidates listed, ascending
  int16_t cand[kDeferCand];
};

struct AssignSmem {
  uint64_t x_full[2], x_free[2], t_full[2], t_free[2];
  uint32_t tmem_base;
  int abort;
  int claim_h, claim_c;
  float max_nrm;
  float max_kap;
  float xq[4][kTileRows];                  // |x|^2 per column quarter's dimensions
  float mq[4][kTileRows];                  // per-quarter maxima of u
  uint8_t kc[4][kTileRows];                // candidates per quarter (saturating)
  int16_t cand[4][kTileRows][kQuarterCand];
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

// grid: min(#SMs, chunks) CTAs, block kAssignThreads. Dynamic smem:
// [AssignSmem][X 2 x 128 x D bf16][nu_hi CP x D][nu_lo CP x D][ones 128 x 16][kappa parts CP x 16]
template <int D, int CP>
__global__ void __launch_bounds__(kAssignThreads, 1)
    assign_kernel(const __grid_constant__ CUtensorMap xmap, int N, int nv, int C, int BH,
                  const uint16_t* __restrict__ nu_hi, const uint16_t* __restrict__ nu_lo,
                  const double* __restrict__ kappa64, const float* __restrict__ nunorm,
                  int32_t* __restrict__ head_next, int32_t* __restrict__ assign,
                  int32_t* __restrict__ defer_count, DeferRec* __restrict__ defer,
                  float* __restrict__ xnorm, int xnorm_mode, float* __restrict__ head_max,
                  int* __restrict__ err) {
  constexpr int kQCols = CP / 4;      // score columns per scorer thread
  constexpr int kLoads = kQCols / 32;  // 32-column TMEM loads per thread
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
  const int nchunk = (ntiles + kChunkTiles - 1) / kChunkTiles;
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

  int i = 0;  // tiles started by this CTA: selects buffers and barrier phases
  int cur_h = -1;
  int h_from = static_cast<int>(static_cast<long long>(blockIdx.x) * BH / gridDim.x);
  while (true) {
    if (tid == 0) {  // claim the next chunk: this head first, then the following ones
      int found = -1, c = 0;
      for (int k = 0; k < BH && found < 0; ++k) {
        const int hh = h_from + k < BH ? h_from + k : h_from + k - BH;
        const int got = atomicAdd(&head_next[hh], 1);
        if (got < nchunk) {
          found = hh;
          c = got;
        }
      }
      S->claim_h = found;
      S->claim_c = c;
    }
    __syncthreads();  // every role is done with the previous chunk
    if (__syncthreads_or(S->claim_h < 0 || *abort)) break;
    const int h = S->claim_h;
    const int t0 = S->claim_c * kChunkTiles, t1 = min(ntiles, t0 + kChunkTiles);
    h_from = h;
    const int row0 = h * N;
    if (h != cur_h) {  // head h: nu_hi, nu_lo into the swizzled K-major layout of the B operand,
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
          head_max[2 * h] = mn;  // for fixup_kernel (every CTA of the head writes the same)
          head_max[2 * h + 1] = mk;
        }
      }
      fence_proxy_async_smem();
      __syncthreads();
      cur_h = h;
    }

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
    } else {
      // ------------------------------------------------------------ scorers
      const int lq = warp & 3;          // TMEM lane quarter
      const int cq = (warp - 1) >> 2;   // column quarter
      const int r = lq * 32 + lane;     // tile row
      const int quad_bar = 1 + lq;
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
        const int tok = tt * kTileRows + r;
        float xsq = 0.f;
        if (xnorm_mode == kXnormLoad) {
          // the scorers never read this X tile: it goes back to the producer at once
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&S->x_free[b]));
          if (tok < nv) xsq = __ldg(xnorm + static_cast<size_t>(h) * nv + tok);
        } else {  // |x|^2 over this quarter of the dimensions; then the X buffer is free
          const uint8_t* xb = xs + b * kXBytes;
          float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
          for (int c = cq * (D / 4); c < (cq + 1) * (D / 4); c += 8) {
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
          S->xq[cq][r] = (a0 + a1) + (a2 + a3);
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&S->x_free[b]));
        }
        // this quarter's scores into registers; then the accumulator is free
        const uint32_t ta = lane_base + b * CP + cq * kQCols;
        float v[kQCols];
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
        named_sync(quad_bar, 128);
        // candidates of this quarter within 2E of the row maximum
        {
          const float U = fmaxf(fmaxf(S->mq[0][r], S->mq[1][r]), fmaxf(S->mq[2][r], S->mq[3][r]));
          if (xnorm_mode != kXnormLoad) {
            xsq = (S->xq[0][r] + S->xq[1][r]) + (S->xq[2][r] + S->xq[3][r]);
            if (xnorm_mode == kXnormStore && cq == 0 && tok < nv) xnorm[static_cast<size_t>(h) * nv + tok] = xsq;
          }
          const float thr = U - ldexpf(sqrtf(xsq) * max_nrm + 0.5f * max_kap, -12);
          int k = 0;
          int16_t cl[kQuarterCand] = {0, 0, 0, 0};
#pragma unroll
          for (int w32 = 0; w32 < kLoads; ++w32) {
            // eight independent partial masks keep the OR chains short
            uint32_t p8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) p8[u] = 0u;
#pragma unroll
            for (int q = 0; q < 32; ++q) p8[q & 7] |= (v[w32 * 32 + q] >= thr ? 1u : 0u) << q;
            uint32_t bw = ((p8[0] | p8[1]) | (p8[2] | p8[3])) | ((p8[4] | p8[5]) | (p8[6] | p8[7]));
            while (bw) {
              const int q = __ffs(bw) - 1;
              bw &= bw - 1;
              if (k < kQuarterCand) cl[k] = static_cast<int16_t>(cq * kQCols + 32 * w32 + q);
              ++k;
            }
          }
          S->kc[cq][r] = static_cast<uint8_t>(min(k, 255));
#pragma unroll
          for (int q = 0; q < kQuarterCand; ++q) S->cand[cq][r][q] = cl[q];
        }
        named_sync(quad_bar, 128);
        if (cq == 0) {  // the row's decision
          int L = -3;   // not a video token
          int total = 0;
          bool listable = true;
          if (tok < nv) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int kq = S->kc[q][r];
              total += kq;
              listable = listable && kq <= kQuarterCand;
              // a padding column (only with non-finite input) is never listed
              for (int u = 0; u < min(kq, kQuarterCand); ++u) listable = listable && S->cand[q][r][u] < C;
            }
            if (total == 1) {
#pragma unroll
              for (int q = 0; q < 4; ++q)
                if (S->kc[q][r] == 1) L = S->cand[q][r][0];
              if (L >= C) L = -2;  // a padding column (only with non-finite input)
            } else {
              L = -1;
            }
          }
          const size_t grp = (static_cast<size_t>(h) * ntiles + tt) * 4 + lq;
          // listed rows get the slots in lane order; the rest are marked -2
          const unsigned dm = __ballot_sync(0xffffffffu, L == -1 && listable && total <= kDeferCand);
          const int slot = __popc(dm & ((1u << lane) - 1u));
          if (L == -1) {
            if (((dm >> lane) & 1u) && slot < kDeferSlots) {
              DeferRec rec;
              rec.tok = tok;
              rec.n = total;
              int n = 0;
#pragma unroll
              for (int q = 0; q < 4; ++q)
                for (int u = 0; u < S->kc[q][r]; ++u) rec.cand[n++] = S->cand[q][r][u];
              for (; n < kDeferCand; ++n) rec.cand[n] = 0;
              defer[grp * kDeferSlots + slot] = rec;
            } else {
              L = -2;  // too many to list: fixup_kernel compares every cluster
            }
          }
          if (L != -3) assign[static_cast<size_t>(h) * nv + tok] = L;
          // listed records (at most kDeferSlots), plus kDeferAll if any row has label -2
          const unsigned all = __ballot_sync(0xffffffffu, L == -2);
          if (lane == 0) defer_count[grp] = min(__popc(dm), kDeferSlots) | (all ? kDeferAll : 0);
        }
      }
    }
    i += t1 - t0;
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

// ---------------------------------------------------------------- fixup
//
// Decides the rows the scorers could not: the listed deferred rows of every
// (tile, 32-row group) and the rows labelled -2. One warp per group; lane l
// holds dimensions (D/32) l .. (D/32) l + D/32 - 1 of the row. First, in fp32,
// t_j = x.(nu_hi + nu_lo)_j - kappa_j / 2: the products are exact, and the
// sums and the rounded -kappa_j/2 err by far less than
// 2^-17 (|x||nu_j| + |kappa_j|), so every j within
// E2 = 2^-16 (|x| max|nu| + max|kappa| / 2) of the best t survives; one
// survivor is the answer; otherwise the survivors are re-scored exactly,
// kappa_j - 2 x.nu_j from the fp64 nu and kappa, ties to the smaller j.
template <int D, int CP>
__device__ float approx_score(const uint16_t* __restrict__ hi, const uint16_t* __restrict__ lo,
                              const double* __restrict__ kap, int j, const float* xv, int lane) {
  constexpr int kPer = D / 32;
  const size_t o = static_cast<size_t>(j) * D + kPer * lane;
  float p = 0.f;
  if (kPer == 4) {
    const uint2 h2 = __ldg(reinterpret_cast<const uint2*>(hi + o));
    const uint2 l2 = __ldg(reinterpret_cast<const uint2*>(lo + o));
    p = fmaf(xv[0], __uint_as_float(h2.x << 16), p);
    p = fmaf(xv[0], __uint_as_float(l2.x << 16), p);
    p = fmaf(xv[1], __uint_as_float(h2.x & 0xffff0000u), p);
    p = fmaf(xv[1], __uint_as_float(l2.x & 0xffff0000u), p);
    p = fmaf(xv[2], __uint_as_float(h2.y << 16), p);
    p = fmaf(xv[2], __uint_as_float(l2.y << 16), p);
    p = fmaf(xv[3], __uint_as_float(h2.y & 0xffff0000u), p);
    p = fmaf(xv[3], __uint_as_float(l2.y & 0xffff0000u), p);
  } else {
    const uint32_t h1 = __ldg(reinterpret_cast<const uint32_t*>(hi + o));
    const uint32_t l1 = __ldg(reinterpret_cast<const uint32_t*>(lo + o));
    p = fmaf(xv[0], __uint_as_float(h1 << 16), p);
    p = fmaf(xv[0], __uint_as_float(l1 << 16), p);
    p = fmaf(xv[1], __uint_as_float(h1 & 0xffff0000u), p);
    p = fmaf(xv[1], __uint_as_float(l1 & 0xffff0000u), p);
  }
  for (int s = 16; s > 0; s >>= 1) p += __shfl_xor_sync(0xffffffffu, p, s);
  return p + static_cast<float>(-0.5 * kap[j]);
}

template <int D>
__device__ __forceinline__ void load_row(const uint16_t* __restrict__ xrow, float* xv, int lane) {
  xv[0] = xv[1] = xv[2] = xv[3] = 0.f;
  if (D == 128) {
    const uint2 w = __ldg(reinterpret_cast<const uint2*>(xrow) + lane);
    xv[0] = __uint_as_float(w.x << 16);
    xv[1] = __uint_as_float(w.x & 0xffff0000u);
    xv[2] = __uint_as_float(w.y << 16);
    xv[3] = __uint_as_float(w.y & 0xffff0000u);
  } else {
    const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(xrow) + lane);
    xv[0] = __uint_as_float(w << 16);
    xv[1] = __uint_as_float(w & 0xffff0000u);
  }
}

// exact score kappa_j - 2 x.nu_j in fp64 (whole warp)
template <int D>
__device__ __forceinline__ double exact_score(const double* __restrict__ nu64h, const double* __restrict__ kap,
                                              int j, const float* xv, int lane) {
  constexpr int kPer = D / 32;
  const double* nj = nu64h + static_cast<size_t>(j) * D + kPer * lane;
  double e = 0.0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) e = fma(static_cast<double>(xv[u]), nj[u], e);
  for (int s = 16; s > 0; s >>= 1) e += __shfl_xor_sync(0xffffffffu, e, s);
  return kap[j] - 2.0 * e;
}

// The label of one row from its listed candidates (n >= 1, ascending): the
// fp32 scores decide when one candidate stays within E2 of the best,
// otherwise the survivors are compared exactly (ties to the smaller j).
template <int D, int CP>
__device__ int decide_listed(const float* xv, const uint16_t* __restrict__ hi, const uint16_t* __restrict__ lo,
                             const double* __restrict__ nu64h, const double* __restrict__ kap, float E2,
                             const int16_t* cand, int n, int lane) {
  float t[kDeferCand];
  float T = -INFINITY;
#pragma unroll
  for (int q = 0; q < kDeferCand; ++q) {
    t[q] = q < n ? approx_score<D, CP>(hi, lo, kap, cand[q], xv, lane) : -INFINITY;
    T = fmaxf(T, t[q]);
  }
  int survivors = 0, only = 0;
#pragma unroll
  for (int q = 0; q < kDeferCand; ++q)
    if (q < n && t[q] >= T - E2) {
      ++survivors;
      only = cand[q];
    }
  if (survivors == 1) return only;
  double best = INFINITY;
  int bj = 0;
#pragma unroll
  for (int q = 0; q < kDeferCand; ++q) {
    if (q >= n || t[q] < T - E2) continue;
    const double sc = exact_score<D>(nu64h, kap, cand[q], xv, lane);
    if (sc < best) {
      best = sc;
      bj = cand[q];
    }
  }
  return bj;
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
    const double* nj = nu64h + static_cast<size_t>(j) * D;
    double e[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
    for (int i = 0; i < D; i += 8) {
      const uint4 xw = __ldg(reinterpret_cast<const uint4*>(xrow + i));
      const uint32_t w[4] = {xw.x, xw.y, xw.z, xw.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const double2 nv = __ldg(reinterpret_cast<const double2*>(nj + i + 2 * u));
        e[u] = fma(static_cast<double>(__uint_as_float(w[u] << 16)), nv.x, e[u]);
        e[u] = fma(static_cast<double>(__uint_as_float(w[u] & 0xffff0000u)), nv.y, e[u]);
      }
    }
    const double sc = kap[j] - 2.0 * ((e[0] + e[1]) + (e[2] + e[3]));
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

// E2 = 2^-16 (|x| max|nu| + max|kappa| / 2) of a row (whole warp)
__device__ __forceinline__ float row_e2(const float* xv, float max_nrm, float max_kap) {
  float xx = xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
  for (int s = 16; s > 0; s >>= 1) xx += __shfl_xor_sync(0xffffffffu, xx, s);
  return ldexpf(sqrtf(xx) * max_nrm + 0.5f * max_kap, -16);
}

// grid: ceil(BH * ntiles * 4 / 8) blocks of 8 warps, one warp per (head, tile, 32-row group)
template <int D, int CP>
__global__ void __launch_bounds__(256)
    fixup_kernel(const uint16_t* __restrict__ x, int N, int nv, int C, int BH, int ntiles,
                 const uint16_t* __restrict__ nu_hi, const uint16_t* __restrict__ nu_lo,
                 const double* __restrict__ nu64, const double* __restrict__ kappa64,
                 const float* __restrict__ head_max, int32_t* __restrict__ assign,
                 const int32_t* __restrict__ defer_count, const DeferRec* __restrict__ defer,
                 int* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  if (timed_out_before(err)) return;  // the scorers may not have written their lists
  const long long grp = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (grp >= static_cast<long long>(BH) * ntiles * 4) return;
  const int dc = defer_count[grp];
  if (dc == 0) return;  // (warp-uniform) nothing was deferred in these 32 rows
  const int n_def = min(dc & (kDeferAll - 1), kDeferSlots);
  const int h = static_cast<int>(grp / (static_cast<long long>(ntiles) * 4));
  const int rem = static_cast<int>(grp - static_cast<long long>(h) * ntiles * 4);
  const int tt = rem >> 2, lq = rem & 3;
  const float mn = head_max[2 * h], mk = head_max[2 * h + 1];
  const uint16_t* hi = nu_hi + static_cast<size_t>(h) * CP * D;
  const uint16_t* lo = nu_lo + static_cast<size_t>(h) * CP * D;
  const double* nuh = nu64 + static_cast<size_t>(h) * C * D;
  const double* kap = kappa64 + static_cast<size_t>(h) * CP;
  int32_t* asg = assign + static_cast<size_t>(h) * nv;
  const uint16_t* xh = x + static_cast<size_t>(h) * N * D;
  // listed rows
  for (int s = 0; s < n_def; ++s) {
    const DeferRec& rec = defer[grp * kDeferSlots + s];
    const int tok = rec.tok;
    if (tok < 0 || tok >= nv) continue;
    const int n = min(max(rec.n, 1), kDeferCand);
    int16_t cand[kDeferCand];
    bool valid = true;  // a list that does not look right falls back to every cluster
#pragma unroll
    for (int q = 0; q < kDeferCand; ++q) {
      cand[q] = rec.cand[q];
      valid = valid && (q >= n || (cand[q] >= 0 && cand[q] < C));
    }
    int lbl;
    if (valid) {
      float xv[4];
      load_row<D>(xh + static_cast<size_t>(tok) * D, xv, lane);
      lbl = decide_listed<D, CP>(xv, hi, lo, nuh, kap, row_e2(xv, mn, mk), cand, n, lane);
    } else {
      lbl = decide_all<D>(xh + static_cast<size_t>(tok) * D, nuh, kap, C, lane);
    }
    if (lane == 0) asg[tok] = lbl;
  }
  // rows whose candidates could not be listed: every cluster
  if (!(dc & kDeferAll)) return;
  const int tok = tt * kTileRows + lq * 32 + lane;
  unsigned all = __ballot_sync(0xffffffffu, tok < nv && asg[tok] == -2);
  while (all) {
    const int l = __ffs(all) - 1;
    all &= all - 1;
    const int t = tt * kTileRows + lq * 32 + l;
    const int lbl = decide_all<D>(xh + static_cast<size_t>(t) * D, nuh, kap, C, lane);
    if (lane == 0) asg[t] = lbl;
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

__device__ __forceinline__ double flushed(float v) {
  return fabsf(v) < 5.9604644775390625e-08f ? 0.0 : static_cast<double>(v);  // 2^-24
}

__device__ __forceinline__ void red_f64(double* dst, double v) {
  asm volatile("red.global.add.f64 [%0], %1;" ::"l"(dst), "d"(v) : "memory");
}

__device__ __forceinline__ void red_s32(int32_t* dst, int v) {
  asm volatile("red.global.add.s32 [%0], %1;" ::"l"(dst), "r"(v) : "memory");
}

// grid (ceil(nv / kUpdTokens), BH), block kUpdThreads. The CTA groups its
// kUpdTokens consecutive tokens by label in shared memory (the order inside a
// cluster is irrelevant: the sums are exact), adds its member counts to
// counts[h][j], and each warp sums a contiguous run of the grouped order in
// fp64, adding every cluster's partial sum to sums[h][j]. The rows it reads
// all lie in the chunk's own contiguous slice of X.
template <int D>
__global__ void __launch_bounds__(kUpdThreads)
    update_kernel(const uint16_t* __restrict__ x, int N, int nv, int C,
                  const int32_t* __restrict__ assign, double* __restrict__ sums,
                  int32_t* __restrict__ counts, int* __restrict__ err) {
  constexpr int kPer = D / 32;
  constexpr int kBatch = 16;
  __shared__ int cnt[kMaxClusters];
  __shared__ int base[kMaxClusters + 1];
  __shared__ int16_t order[kUpdTokens];
  const int h = blockIdx.y, c0 = blockIdx.x * kUpdTokens;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (timed_out_before(err)) return;  // labels of an aborted step are not to be trusted
  const int n = min(kUpdTokens, nv - c0);
  const int32_t* a = assign + static_cast<size_t>(h) * nv + c0;
  for (int j = tid; j < C; j += kUpdThreads) cnt[j] = 0;
  __syncthreads();
  for (int t = tid; t < n; t += kUpdThreads) {
    const int l = a[t];
    if (l >= 0 && l < C) atomicAdd(&cnt[l], 1);
    else report_error(err, kErrBadLabel);
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the counts
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
    if (cnt[j] > 0) red_s32(&counts[static_cast<size_t>(h) * C + j], cnt[j]);
  }
  __syncthreads();
  for (int j = tid; j < C; j += kUpdThreads) cnt[j] = 0;
  __syncthreads();
  for (int t = tid; t < n; t += kUpdThreads) {
    const int l = a[t];
    if (l >= 0 && l < C) order[base[l] + atomicAdd(&cnt[l], 1)] = static_cast<int16_t>(t);
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
  double acc[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) acc[u] = 0.0;
  bool any = false;
  auto flush = [&]() {
    if (any) {
      double* dst = sums + (static_cast<size_t>(h) * C + j) * D + kPer * lane;
#pragma unroll
      for (int u = 0; u < kPer; ++u) red_f64(dst + u, acc[u]);
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) acc[u] = 0.0;
    any = false;
  };
  for (int pb = p0; pb < p1; pb += kBatch) {
    uint32_t w0[kBatch], w1[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {  // the batch's rows in flight together
      w0[q] = 0u;
      w1[q] = 0u;
      if (pb + q < p1) {
        const int t = order[pb + q];
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
      acc[0] += flushed(__uint_as_float(w0[q] << 16));
      acc[1] += flushed(__uint_as_float(w0[q] & 0xffff0000u));
      if (kPer == 4) {
        acc[2] += flushed(__uint_as_float(w1[q] << 16));
        acc[3] += flushed(__uint_as_float(w1[q] & 0xffff0000u));
      }
      any = true;
    }
  }
  flush();
}

// ---------------------------------------------------------------- finalize

// grid (C, BH), block d: centroid = fp32(sum / n) (IEEE fp64 division, one
// rounding), an empty cluster keeps its centroid; clears the sums and the
// chunk counters for the next half-step.
__global__ void finalize_kernel(double* __restrict__ sums, int32_t* __restrict__ counts,
                                float* __restrict__ cent, int32_t* __restrict__ sizes,
                                int32_t* __restrict__ head_next, int C, int d) {
  const int h = blockIdx.y, j = blockIdx.x, i = threadIdx.x;
  const int n = counts[h * C + j];
  const size_t e = (static_cast<size_t>(h) * C + j) * d + i;
  if (n > 0) cent[e] = static_cast<float>(sums[e] / static_cast<double>(n));
  sums[e] = 0.0;
  __syncthreads();
  if (i == 0) {
    sizes[h * C + j] = n;
    counts[h * C + j] = 0;
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
  float* kappa;
  float* nunorm;
  double* sums;
  int32_t* counts;
  int32_t* head_next;
  float* head_max;
  float* xnorm;
  int32_t* defer_count;
  DeferRec* defer;
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
  w.kappa = cv.take<float>(static_cast<size_t>(BH) * CP);
  w.nunorm = cv.take<float>(static_cast<size_t>(BH) * CP);
  w.sums = cv.take<double>(static_cast<size_t>(BH) * Cmax * d);
  w.counts = cv.take<int32_t>(static_cast<size_t>(BH) * Cmax);
  w.head_next = cv.take<int32_t>(static_cast<size_t>(BH));
  w.head_max = cv.take<float>(static_cast<size_t>(BH) * 2);
  w.xnorm = cv.take<float>(static_cast<size_t>(BH) * nv);
  w.defer_count = cv.take<int32_t>(static_cast<size_t>(BH) * ntiles * 4);
  w.defer = cv.take<DeferRec>(static_cast<size_t>(BH) * ntiles * 4 * kDeferSlots);
  if (out) *out = w;
  return cv.used + 256;
}

template <int D, int CP>
svoo_status launch_assign(const CUtensorMap& xmap, const svoo_shape* sh, const void* x, int C,
                          const StepWs& w, int32_t* assign, float* xnorm, int xnorm_mode,
                          int32_t* dev_err, cudaStream_t st) {
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
  const int ntiles = (nv + kTileRows - 1) / kTileRows;
  const long long chunks = static_cast<long long>(BH) * ((ntiles + kChunkTiles - 1) / kChunkTiles);
  const int grid = static_cast<int>(chunks < sms ? chunks : sms);
  assign_kernel<D, CP><<<grid, kAssignThreads, smem, st>>>(
      xmap, N, nv, C, BH, w.nu_hi, w.nu_lo, w.kappa64, w.nunorm, w.head_next, assign,
      w.defer_count, w.defer, xnorm, xnorm_mode, w.head_max, dev_err);
  if (cudaGetLastError() != cudaSuccess) return SVOO_ERR_CUDA;
  const long long groups = static_cast<long long>(BH) * ntiles * 4;
  fixup_kernel<D, CP><<<static_cast<unsigned>((groups + 7) / 8), 256, 0, st>>>(
      static_cast<const uint16_t*>(x), N, nv, C, BH, ntiles, w.nu_hi, w.nu_lo, w.nu64, w.kappa64,
      w.head_max, assign, w.defer_count, w.defer, dev_err);
  if (cudaGetLastError() != cudaSuccess) return SVOO_ERR_CUDA;
  update_kernel<D><<<dim3((nv + kUpdTokens - 1) / kUpdTokens, BH), kUpdThreads, 0, st>>>(
      static_cast<const uint16_t*>(x), N, nv, C, assign, w.sums, w.counts, dev_err);
  return SVOO_OK;
}

// One half-step. metric_cent == nullptr: identity metric. xnorm: per-token
// |x|^2 store of this side (xnorm_mode kXnormStore / kXnormLoad), else the
// step computes |x|^2 itself.
svoo_status run_step(const svoo_shape* sh, const void* x, int C, float* cent, int32_t* sizes,
                     int32_t* assign, const float* metric_cent, const int32_t* metric_sizes,
                     int metric_C, const StepWs& w, int32_t* dev_err, cudaStream_t st,
                     int zero_C, float* xnorm = nullptr, int xnorm_mode = kXnormCompute) {
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
  metric_nu_kernel<<<dim3(CP / 32, BH), 128, metric_nu_smem(d), st>>>(
      metric_cent ? w.M : nullptr, cent, C, CP, d, w.nu64, w.nu_hi, w.nu_lo, w.kappa64, w.kappa,
      w.nunorm);
  CUtensorMap xmap;
  if (encode_tiled_2d(&xmap, x, static_cast<uint64_t>(BH) * N, d, kTileRows, 64) != CUDA_SUCCESS)
    return SVOO_ERR_CUDA;
  if (!xnorm) {  // a lone half-step computes |x|^2 from the tiles
    xnorm = w.xnorm;
    xnorm_mode = kXnormCompute;
  }
  svoo_status s;
  if (d == 128)
    s = CP == 256 ? launch_assign<128, 256>(xmap, sh, x, C, w, assign, xnorm, xnorm_mode, dev_err, st)
                  : launch_assign<128, 128>(xmap, sh, x, C, w, assign, xnorm, xnorm_mode, dev_err, st);
  else
    s = CP == 256 ? launch_assign<64, 256>(xmap, sh, x, C, w, assign, xnorm, xnorm_mode, dev_err, st)
                  : launch_assign<64, 128>(xmap, sh, x, C, w, assign, xnorm, xnorm_mode, dev_err, st);
  if (s != SVOO_OK) return s;
  finalize_kernel<<<dim3(C, BH), d, 0, st>>>(w.sums, w.counts, cent, sizes, w.head_next, C, d);
  return launch_status();
}

bool cluster_counts_ok(int C) { return C >= 1 && C <= 256; }

// Workspace of a whole svoo_cluster call: one half-step's scratch, then the
// per-token |x|^2 of the queries and of the keys (fp32 [BH][N - n_text] each).
size_t carve_call(void* ws, const svoo_shape* sh, int Cmax, StepWs* w, float** xn_q, float** xn_k) {
  const size_t step = carve_step(ws, bh_of(sh), sh->d, Cmax, nvideo_of(sh), w);
  Carver cv(ws ? static_cast<char*>(ws) + step : nullptr);
  const size_t n = static_cast<size_t>(bh_of(sh)) * nvideo_of(sh);
  float* a = cv.take<float>(n);
  float* b = cv.take<float>(n);
  if (xn_q) *xn_q = a;
  if (xn_k) *xn_k = b;
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
  return carve_call(nullptr, shape, n_qc > n_kc ? n_qc : n_kc, nullptr, nullptr, nullptr);
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
  size_t need = carve_call(workspace, shape, n_qc > n_kc ? n_qc : n_kc, &w, &xn_q, &xn_k);
  if (workspace_bytes < need) return SVOO_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!warm) {
    init_centroids_kernel<<<dim3(n_qc, BH), d, 0, st>>>(static_cast<const uint16_t*>(q), N, nv, d, n_qc, q_cent);
    init_centroids_kernel<<<dim3(n_kc, BH), d, 0, st>>>(static_cast<const uint16_t*>(k), N, nv, d, n_kc, k_cent);
  }
  const int Cmax = n_qc > n_kc ? n_qc : n_kc;
  for (int it = 0; it < iters; ++it) {
    const bool ident = identity || (it == 0 && !warm);
    const int xmode = it == 0 ? kXnormStore : kXnormLoad;  // inputs fixed for the whole call
    svoo_status s = run_step(shape, q, n_qc, q_cent, q_sizes, q_assign, ident ? nullptr : k_cent,
                             k_sizes, n_kc, w, dev_err, st, it == 0 ? Cmax : 0, xn_q, xmode);
    if (s != SVOO_OK) return s;
    s = run_step(shape, k, n_kc, k_cent, k_sizes, k_assign, identity ? nullptr : q_cent, q_sizes,
                 n_qc, w, dev_err, st, 0, xn_k, xmode);
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
