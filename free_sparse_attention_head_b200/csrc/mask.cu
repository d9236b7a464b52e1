// mask.cu -- cluster-pair block mask and tail merging.
//
// pair_mass_kernel  estimated attention mass of every (query cluster a, key
//                   cluster b) pair from the centroids (PSA section 2 on
//                   SVG2's centroid scores and top-k cluster selection; iCATS
//                   section 4's cluster-level scores):
//                     s_ab = scale * mu_a . c_b, m_a = max_{n_b > 0} s_ab,
//                     Z_a = sum_b n_b e^{s_ab - m_a},
//                     w_ab = n_a * (n_b e^{s_ab - m_a}) / Z_a,
//                   fp32 with a fixed operation order (sequential fmaf dot
//                   product and sum), so the kept set is reproducible bit for
//                   bit; e^x is the library's own Cody-Waite + Taylor exp.
// select_kernel     keeps the top pairs of the order (per-cluster best,
//                   w desc, a asc, b asc) by an MSB-first radix select over
//                   64-bit keys: the K-th key (keep ratio) or the key where
//                   the fixed-point mass reaches ceil(p * total) (top-p).
// tail_merge_kernel iCATS section 4.3 / appendix E.1: identical-mask merge,
//                   then rounds of mutually nearest tail moves.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace svoo {

constexpr int kMassRows = 8;

// e^x for x <= 0 (x < -87 gives 0): n = rint(x log2 e); r = x - n ln2 by
// Cody & Waite's two-constant reduction (ln2_hi = 22713 / 2^15, ln2_lo =
// fp32(ln 2 - ln2_hi)); e^r by the degree-7 Taylor polynomial in Horner form;
// the result scaled by 2^n built from its exponent bits. Every step is one
// explicitly rounded fp32 operation.
__device__ __forceinline__ float exp_own(float x) {
  const float log2e = 1.4426950408889634f;
  const float ln2_hi = 22713.0f / 32768.0f;
  const float ln2_lo = static_cast<float>(0.69314718055994530942 - 22713.0 / 32768.0);
  const float c2 = static_cast<float>(1.0 / 2.0), c3 = static_cast<float>(1.0 / 6.0);
  const float c4 = static_cast<float>(1.0 / 24.0), c5 = static_cast<float>(1.0 / 120.0);
  const float c6 = static_cast<float>(1.0 / 720.0), c7 = static_cast<float>(1.0 / 5040.0);
  if (!(x >= -87.0f)) return 0.0f;
  float t = __fmul_rn(x, log2e);
  float n = rintf(t);
  float r = __fmaf_rn(-n, ln2_hi, x);
  r = __fmaf_rn(-n, ln2_lo, r);
  float p = c7;
  p = __fmaf_rn(p, r, c6);
  p = __fmaf_rn(p, r, c5);
  p = __fmaf_rn(p, r, c4);
  p = __fmaf_rn(p, r, c3);
  p = __fmaf_rn(p, r, c2);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  int ni = static_cast<int>(n);
  float s = __uint_as_float(static_cast<uint32_t>(ni + 127) << 23);
  return __fmul_rn(p, s);
}

// grid (ceil(Cq / 8), BH), block 256: thread b owns key cluster b (Ck <= 256).
__global__ void __launch_bounds__(256)
    pair_mass_kernel(const float* __restrict__ q_cent, const float* __restrict__ k_cent,
                     const int32_t* __restrict__ q_sizes, const int32_t* __restrict__ k_sizes,
                     int Cq, int Ck, int d, float scale, float* __restrict__ w,
                     int32_t* __restrict__ top1) {
  __shared__ float mu[kMassRows][128];
  __shared__ float e_s[kMassRows][256];
  __shared__ float red_f[kMassRows][8];
  __shared__ int red_i[kMassRows][8];
  __shared__ float m_s[kMassRows], z_s[kMassRows];
  const int h = blockIdx.y, a0 = blockIdx.x * kMassRows, b = threadIdx.x;
  const int lane = b & 31, warp = b >> 5;
  for (int e = threadIdx.x; e < kMassRows * d; e += blockDim.x) {
    int r = e / d, c = e % d;
    mu[r][c] = (a0 + r < Cq) ? q_cent[(static_cast<size_t>(h) * Cq + a0 + r) * d + c] : 0.f;
  }
  __syncthreads();
  const bool live_b = b < Ck;
  const int nb = live_b ? k_sizes[h * Ck + b] : 0;
  float s[kMassRows];
#pragma unroll
  for (int r = 0; r < kMassRows; ++r) s[r] = 0.f;
  if (live_b) {
    const float* cb = k_cent + (static_cast<size_t>(h) * Ck + b) * d;
    for (int i = 0; i < d; ++i) {
      float c = __ldg(cb + i);
#pragma unroll
      for (int r = 0; r < kMassRows; ++r) s[r] = __fmaf_rn(mu[r][i], c, s[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < kMassRows; ++r) {
    s[r] = __fmul_rn(scale, s[r]);
    float v = (live_b && nb > 0) ? s[r] : -INFINITY;
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    if (lane == 0) red_f[r][warp] = v;
  }
  __syncthreads();
  if (threadIdx.x < kMassRows) {
    float v = -INFINITY;
    for (int ww = 0; ww < 8; ++ww) v = fmaxf(v, red_f[threadIdx.x][ww]);
    m_s[threadIdx.x] = v;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMassRows; ++r)
    e_s[r][b] = (live_b && nb > 0) ? exp_own(__fsub_rn(s[r], m_s[r])) : 0.f;
  __syncthreads();
  if (threadIdx.x < kMassRows) {  // Z_a in ascending b, one fmaf per term
    float z = 0.f;
    for (int bb = 0; bb < Ck; ++bb)
      z = __fmaf_rn(static_cast<float>(k_sizes[h * Ck + bb]), e_s[threadIdx.x][bb], z);
    z_s[threadIdx.x] = z;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kMassRows; ++r) {
    const int a = a0 + r;
    float wab = 0.f;
    if (a < Cq && live_b) {
      float na = static_cast<float>(q_sizes[h * Cq + a]);
      float t = __fmul_rn(static_cast<float>(nb), e_s[r][b]);
      float u = __fmul_rn(na, t);
      float z = z_s[r];
      wab = z > 0.f ? __fdiv_rn(u, z) : 0.f;
      w[(static_cast<size_t>(h) * Cq + a) * Ck + b] = wab;
    }
    // argmax over b, ties to the lower b
    float bv = live_b ? wab : -1.f;
    int bi = live_b ? b : 0x7fffffff;
    for (int o = 16; o > 0; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      red_f[r][warp] = bv;
      red_i[r][warp] = bi;
    }
  }
  __syncthreads();
  if (threadIdx.x < kMassRows && a0 + threadIdx.x < Cq) {
    const int r = threadIdx.x;
    float bv = red_f[r][0];
    int bi = red_i[r][0];
    for (int ww = 1; ww < 8; ++ww) {
      if (red_f[r][ww] > bv || (red_f[r][ww] == bv && red_i[r][ww] < bi)) {
        bv = red_f[r][ww];
        bi = red_i[r][ww];
      }
    }
    top1[h * Cq + a0 + r] = bi;
  }
}

// Sort key of pair (a, b): larger = earlier in the selection order.
__device__ __forceinline__ uint64_t pair_key(float wv, bool forced, int a, int b) {
  uint64_t wb = static_cast<uint64_t>(__float_as_uint(wv) & 0x7fffffffu);
  return (static_cast<uint64_t>(forced) << 63) | (wb << 32) |
         (static_cast<uint64_t>(0xffff - a) << 16) | static_cast<uint64_t>(0xffff - b);
}

__device__ __forceinline__ long long mass_fixed(float wv) {
  return static_cast<long long>(floor(static_cast<double>(wv) * 4294967296.0));
}

// One CTA per head, 1024 threads.
__global__ void __launch_bounds__(1024)
    select_kernel(const float* __restrict__ w, const int32_t* __restrict__ top1,
                  const float* __restrict__ keep, int Cq, int Ck, int mode, int has_text, int W,
                  uint64_t* __restrict__ kmask, int32_t* __restrict__ stats) {
  __shared__ unsigned int hist_c[256];
  __shared__ unsigned long long hist_m[256];
  __shared__ int top1_s[256];
  __shared__ unsigned long long sh_prefix, sh_total;
  __shared__ long long sh_rank;
  __shared__ int sh_none;
  __shared__ int kept_count;
  const int h = blockIdx.x, tid = threadIdx.x;
  const int P = Cq * Ck;
  const float* wh = w + static_cast<size_t>(h) * P;
  for (int a = tid; a < Cq; a += blockDim.x) top1_s[a] = top1[h * Cq + a];
  if (tid == 0) {
    sh_prefix = 0;
    sh_total = 0;
    sh_none = 0;
    kept_count = 0;
  }
  __syncthreads();
  const float kv = keep[h];
  long long rank;  // keep mode: rank of the threshold key; top-p: mass still needed
  if (mode == 0) {
    float kf = ceilf(__fmul_rn(kv, static_cast<float>(P)));
    long long K = static_cast<long long>(kf);
    if (K > P) K = P;
    if (K < Cq) K = Cq;
    rank = K;
  } else {
    unsigned long long part = 0;
    for (int idx = tid; idx < P; idx += blockDim.x) part += static_cast<unsigned long long>(mass_fixed(wh[idx]));
    atomicAdd(&sh_total, part);
    __syncthreads();
    long long target = static_cast<long long>(ceil(static_cast<double>(kv) * static_cast<double>(sh_total)));
    rank = target;
    if (target <= 0 && tid == 0) sh_none = 1;
  }
  if (tid == 0) sh_rank = rank;
  __syncthreads();
  if (!sh_none) {
    for (int pass = 0; pass < 8; ++pass) {
      const int shift = 56 - 8 * pass;
      const unsigned long long hi_mask = pass == 0 ? 0ull : (~0ull << (shift + 8));
      for (int i = tid; i < 256; i += blockDim.x) {
        hist_c[i] = 0;
        hist_m[i] = 0;
      }
      __syncthreads();
      const unsigned long long prefix = sh_prefix;
      for (int idx = tid; idx < P; idx += blockDim.x) {
        int a = idx / Ck, b = idx - a * Ck;
        float wv = wh[idx];
        uint64_t key = pair_key(wv, top1_s[a] == b, a, b);
        if ((key & hi_mask) != prefix) continue;
        int dg = static_cast<int>((key >> shift) & 255);
        if (mode == 0) atomicAdd(&hist_c[dg], 1u);
        else atomicAdd(&hist_m[dg], static_cast<unsigned long long>(mass_fixed(wv)));
      }
      __syncthreads();
      if (tid == 0) {
        long long need = sh_rank, cum = 0;
        int chosen = 0;
        for (int dg = 255; dg >= 0; --dg) {
          long long c = mode == 0 ? static_cast<long long>(hist_c[dg]) : static_cast<long long>(hist_m[dg]);
          if (cum + c >= need) {
            chosen = dg;
            break;
          }
          cum += c;
        }
        sh_rank = need - cum;
        sh_prefix = prefix | (static_cast<unsigned long long>(chosen) << shift);
      }
      __syncthreads();
    }
  }
  const unsigned long long T = sh_none ? ~0ull : sh_prefix;
  const int rows = Cq + (has_text ? 1 : 0);
  for (int e = tid; e < rows * W; e += blockDim.x) {
    const int a = e / W, wd = e % W;
    uint64_t bits = 0;
    if (a < Cq) {
      for (int bb = 0; bb < 64; ++bb) {
        const int b = wd * 64 + bb;
        if (b >= Ck) break;
        float wv = wh[a * Ck + b];
        bool forced = top1_s[a] == b;
        if (forced || pair_key(wv, forced, a, b) >= T) bits |= 1ull << bb;
      }
      atomicAdd(&kept_count, __popcll(bits));
      if (has_text && Ck / 64 == wd) bits |= 1ull << (Ck % 64);
    } else {
      for (int bb = 0; bb < 64; ++bb)
        if (wd * 64 + bb <= Ck) bits |= 1ull << bb;
    }
    kmask[(static_cast<size_t>(h) * rows + a) * W + wd] = bits;
  }
  __syncthreads();
  if (tid == 0) stats[h * 8 + 0] = kept_count;
}

// One CTA per head, 1024 threads. In: kmask (select output), cluster sizes and
// labels. Out: merged kmask (in place), q_label [BH][N], merged q_sizes [BH][Gq], stats.
__global__ void __launch_bounds__(1024)
    tail_merge_kernel(uint64_t* __restrict__ kmask, const int32_t* __restrict__ q_sizes_in,
                      const int32_t* __restrict__ q_assign, int N, int nv, int Cq, int W,
                      int has_text, int block_q, int rounds, int32_t* __restrict__ q_label,
                      int32_t* __restrict__ q_sizes_out, int32_t* __restrict__ stats,
                      int* __restrict__ err) {
  constexpr int kMaxW = 5;
  __shared__ uint64_t msk[256][kMaxW];
  __shared__ int sz[256], nsz[256], rep[256], tl[256], nearv[256];
  __shared__ int mv_donor[128], mv_recv[128], mv_cnt[128];
  __shared__ int slot_of[256], quota[128];
  __shared__ int wcnt[32][128];  // per warp of a chunk: tokens of each move's donor
  __shared__ int n_moves, st_ident, st_r[2], st_moved, tiles_before, left;
  const int h = blockIdx.x, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
  const int rows = Cq + (has_text ? 1 : 0);
  uint64_t* km = kmask + static_cast<size_t>(h) * rows * W;
  for (int e = tid; e < Cq * W; e += blockDim.x) msk[e / W][e % W] = km[e];
  for (int a = tid; a < Cq; a += blockDim.x) {
    sz[a] = q_sizes_in[h * Cq + a];
    nsz[a] = 0;
  }
  for (int a = tid; a < 256; a += blockDim.x) slot_of[a] = -1;
  if (tid == 0) {
    st_ident = 0;
    st_r[0] = st_r[1] = 0;
    st_moved = 0;
    tiles_before = 0;
  }
  __syncthreads();
  // (i) identical masks -> lowest non-empty id
  for (int a = tid; a < Cq; a += blockDim.x) {
    int r = a;
    if (sz[a] > 0) {
      for (int a2 = 0; a2 < a; ++a2) {
        if (sz[a2] == 0) continue;
        bool eq = true;
        for (int wd = 0; wd < W; ++wd) eq = eq && (msk[a2][wd] == msk[a][wd]);
        if (eq) {
          r = a2;
          break;
        }
      }
    }
    rep[a] = r;
    atomicAdd(&tiles_before, (sz[a] + block_q - 1) / block_q);
  }
  __syncthreads();
  int32_t* lab = q_label + static_cast<size_t>(h) * N;
  const int32_t* asg = q_assign + static_cast<size_t>(h) * nv;
  for (int i = tid; i < nv; i += blockDim.x) {
    int l = asg[i];
    if (l < 0 || l >= Cq) {
      report_error(err, kErrBadLabel);
      l = 0;
    }
    lab[i] = rep[l];
  }
  for (int i = nv + tid; i < N; i += blockDim.x) lab[i] = Cq;
  for (int a = tid; a < Cq; a += blockDim.x) {
    atomicAdd(&nsz[rep[a]], sz[a]);
    if (rep[a] != a) atomicAdd(&st_ident, 1);
  }
  __syncthreads();
  for (int a = tid; a < Cq; a += blockDim.x) sz[a] = nsz[a];
  __syncthreads();
  // (ii) rounds of mutually nearest tail moves
  for (int round = 0; round < rounds; ++round) {
    for (int a = tid; a < Cq; a += blockDim.x) tl[a] = sz[a] % block_q;
    if (tid == 0) n_moves = 0;
    __syncthreads();
    for (int a = tid; a < Cq; a += blockDim.x) {
      int best = 0x7fffffff, nb = -1;
      if (tl[a] > 0) {
        for (int b = 0; b < Cq; ++b) {
          if (b == a || tl[b] == 0 || tl[a] + tl[b] > block_q) continue;
          int hm = 0;
          for (int wd = 0; wd < W; ++wd) hm += __popcll(msk[a][wd] ^ msk[b][wd]);
          if (hm < best) {
            best = hm;
            nb = b;
          }
        }
      }
      nearv[a] = nb;
    }
    __syncthreads();
    for (int a = tid; a < Cq; a += blockDim.x) {
      int b = nearv[a];
      if (b <= a || nearv[b] != a) continue;
      int donor = tl[a] < tl[b] ? a : b;
      int recv = donor == a ? b : a;
      int cnt = tl[donor];
      int slot = atomicAdd(&n_moves, 1);
      mv_donor[slot] = donor;
      mv_recv[slot] = recv;
      mv_cnt[slot] = cnt;
      sz[recv] += cnt;
      sz[donor] -= cnt;
      for (int wd = 0; wd < W; ++wd) msk[recv][wd] |= msk[donor][wd];
      atomicAdd(&st_r[round < 1 ? 0 : 1], 1);
      atomicAdd(&st_moved, cnt);
    }
    __syncthreads();
    // move the donors' highest-index tail tokens: one backward pass over the
    // labels in chunks of blockDim.x tokens serves every move of the round;
    // thread t of a chunk holds the chunk's t-th highest token, so a token's
    // rank among its donor's tokens is the count in earlier warps plus the
    // count in earlier lanes of its own warp
    const int nm = n_moves;
    for (int m = tid; m < nm; m += blockDim.x) {
      slot_of[mv_donor[m]] = m;
      quota[m] = mv_cnt[m];
    }
    __syncthreads();
    for (int top = nv - 1; top >= 0; top -= blockDim.x) {
      if (tid == 0) left = 0;
      for (int e = tid; e < nwarps * nm; e += blockDim.x) wcnt[e / nm][e % nm] = 0;
      __syncthreads();
      const int i = top - tid;
      int sl = -1;
      if (i >= 0) {
        const int l = lab[i];
        if (l >= 0 && l < Cq) sl = slot_of[l];
      }
      if (sl >= 0 && quota[sl] == 0) sl = -1;
      const unsigned peers = __match_any_sync(0xffffffffu, sl);
      const int rank_w = __popc(peers & ((1u << lane) - 1u));
      if (sl >= 0 && rank_w == 0) wcnt[warp][sl] = __popc(peers);
      __syncthreads();
      if (sl >= 0) {
        int before = rank_w;
        for (int w2 = 0; w2 < warp; ++w2) before += wcnt[w2][sl];
        if (before < quota[sl]) lab[i] = mv_recv[sl];
      }
      __syncthreads();
      for (int m = tid; m < nm; m += blockDim.x) {
        int tot = 0;
        for (int w2 = 0; w2 < nwarps; ++w2) tot += wcnt[w2][m];
        quota[m] = max(0, quota[m] - tot);
        if (quota[m] > 0) left = 1;
      }
      __syncthreads();
      if (!left) break;
    }
    for (int m = tid; m < nm; m += blockDim.x) slot_of[mv_donor[m]] = -1;
    __syncthreads();
  }
  for (int e = tid; e < Cq * W; e += blockDim.x) km[e] = msk[e / W][e % W];
  int32_t* so = q_sizes_out + static_cast<size_t>(h) * rows;
  for (int a = tid; a < Cq; a += blockDim.x) so[a] = sz[a];
  if (has_text && tid == 0) so[Cq] = N - nv;
  __syncthreads();
  if (tid == 0) {
    int ne = 0, after = 0;
    for (int a = 0; a < Cq; ++a) {
      ne += sz[a] > 0;
      after += (sz[a] + block_q - 1) / block_q;
    }
    int32_t* s = stats + h * 8;
    s[1] = ne;
    s[2] = st_ident;
    s[3] = st_r[0];
    s[4] = st_r[1];
    s[5] = tiles_before;
    s[6] = after;
    s[7] = st_moved;
  }
}

}  // namespace svoo

using namespace svoo;

extern "C" size_t svoo_mask_workspace_size(const svoo_shape* shape, int n_qc, int n_kc) {
  if (!shape_ok(shape) || n_qc < 1 || n_qc > 256 || n_kc < 1 || n_kc > 256) return 0;
  Carver cv(nullptr);
  cv.take<float>(static_cast<size_t>(bh_of(shape)) * n_qc * n_kc);
  cv.take<int32_t>(static_cast<size_t>(bh_of(shape)) * n_qc);
  return cv.used + 256;
}

extern "C" svoo_status svoo_build_mask(const svoo_shape* shape, const float* q_cent,
                                       const float* k_cent, const int32_t* q_sizes,
                                       const int32_t* k_sizes, const int32_t* q_assign,
                                       const float* keep, int n_qc, int n_kc, int select_mode,
                                       int block_q, int merge_rounds, float scale,
                                       const svoo_plan* plan, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_err, void* stream) {
  if (!shape_ok(shape) || !q_cent || !k_cent || !q_sizes || !k_sizes || !q_assign || !keep || !plan ||
      !workspace)
    return SVOO_ERR_INVALID_ARG;
  if (!plan->kmask || !plan->q_label || !plan->q_sizes || !plan->stats) return SVOO_ERR_INVALID_ARG;
  if (n_qc < 1 || n_qc > 256 || n_kc < 1 || n_kc > 256) return SVOO_ERR_INVALID_ARG;
  if (select_mode != 0 && select_mode != 1) return SVOO_ERR_INVALID_ARG;
  if (block_q != 64 && block_q != 128) return SVOO_ERR_INVALID_ARG;
  if (merge_rounds < 0 || merge_rounds > 8) return SVOO_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return SVOO_ERR_INVALID_ARG;
  if (workspace_bytes < svoo_mask_workspace_size(shape, n_qc, n_kc)) return SVOO_ERR_WORKSPACE;
  const int BH = bh_of(shape), d = shape->d, W = mask_words(shape, n_kc);
  const int has_text = shape->n_text > 0;
  Carver cv(workspace);
  float* w = cv.take<float>(static_cast<size_t>(BH) * n_qc * n_kc);
  int32_t* top1 = cv.take<int32_t>(static_cast<size_t>(BH) * n_qc);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  pair_mass_kernel<<<dim3((n_qc + kMassRows - 1) / kMassRows, BH), 256, 0, st>>>(
      q_cent, k_cent, q_sizes, k_sizes, n_qc, n_kc, d, scale, w, top1);
  select_kernel<<<BH, 1024, 0, st>>>(w, top1, keep, n_qc, n_kc, select_mode, has_text, W, plan->kmask,
                                     plan->stats);
  tail_merge_kernel<<<BH, 1024, 0, st>>>(plan->kmask, q_sizes, q_assign, shape->N, nvideo_of(shape), n_qc,
                                         W, has_text, block_q, merge_rounds, plan->q_label,
                                         plan->q_sizes, plan->stats, dev_err);
  return launch_status();
}
