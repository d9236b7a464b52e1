// permute.cu -- token permutation into cluster order (PSA section 2 on SVG2's
// semantic-aware permutation), the query tile table and the gathered Q, K, V.
//
// sort_kernel   stable counting sort of one side's labels per head: each of 32
//               warps histograms a contiguous slice, the per-(warp, group)
//               bases come from an exclusive scan, and each warp then walks its
//               slice in order, ranking equal labels inside a 32-token chunk
//               with __match_any_sync -- so ties keep token order and the
//               result is deterministic.
// tiles_kernel  query tiles of at most block_q rows per group, in (group,
//               tile) order, with the group's kept key length; and the
//               attention work units (up to 256 rows of one group).
// gather_kernel dst[p] = src[perm[p]] row copies (16-byte vectors).
#include "common.cuh"
#include "internal.h"

namespace svoo {

constexpr int kSortWarps = 32;
constexpr int kMaxGroups = 264;

// grid (BH, 2): y = 0 sorts query labels (plan q_label, Gq groups), y = 1 key
// labels (k_assign for video tokens, group n_kc for text tokens, Gk groups).
__global__ void __launch_bounds__(kSortWarps * 32)
    sort_kernel(const int32_t* __restrict__ q_label, const int32_t* __restrict__ k_assign, int N,
                int nv, int Gq, int Gk, int n_kc, int32_t* __restrict__ q_perm,
                int32_t* __restrict__ q_off, int32_t* __restrict__ k_perm,
                int32_t* __restrict__ k_off, int* __restrict__ err) {
  __shared__ int hist[kSortWarps][kMaxGroups];
  __shared__ int off_s[kMaxGroups + 1];
  const int h = blockIdx.x, side = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = side == 0 ? Gq : Gk;
  int32_t* perm = (side == 0 ? q_perm : k_perm) + static_cast<size_t>(h) * N;
  int32_t* off = side == 0 ? q_off + static_cast<size_t>(h) * (Gq + 1) : k_off + static_cast<size_t>(h) * (Gk + 1);
  const int32_t* ql = q_label + static_cast<size_t>(h) * N;
  const int32_t* ka = k_assign + static_cast<size_t>(h) * nv;
  auto label_of = [&](int i) -> int {
    int l;
    if (side == 0) l = ql[i];
    else l = i < nv ? ka[i] : n_kc;
    if (l < 0 || l >= G) {
      report_error(err, kErrBadLabel);
      l = G - 1;
    }
    return l;
  };
  for (int e = tid; e < kSortWarps * kMaxGroups; e += blockDim.x) (&hist[0][0])[e] = 0;
  __syncthreads();
  const int slice = ((N + kSortWarps - 1) / kSortWarps + 31) / 32 * 32;
  const int beg = min(N, warp * slice), end = min(N, beg + slice);
  for (int i = beg + lane; i < end; i += 32) atomicAdd(&hist[warp][label_of(i)], 1);
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int g = 0; g < G; ++g) {
      off_s[g] = run;
      int tot = 0;
      for (int w = 0; w < kSortWarps; ++w) tot += hist[w][g];
      run += tot;
    }
    off_s[G] = run;
  }
  __syncthreads();
  for (int g = tid; g < G; g += blockDim.x) {
    int run = off_s[g];
    for (int w = 0; w < kSortWarps; ++w) {
      int c = hist[w][g];
      hist[w][g] = run;
      run += c;
    }
  }
  for (int g = tid; g <= G; g += blockDim.x) off[g] = off_s[g];
  __syncthreads();
  const unsigned lt = (1u << lane) - 1u;
  for (int c0 = beg; c0 < end; c0 += 32) {
    const int i = c0 + lane;
    const bool valid = i < end;
    const int l = valid ? label_of(i) : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, l);
    const int rank = __popc(peers & lt);
    if (valid) perm[hist[warp][l] + rank] = i;
    __syncwarp();
    if (valid && (peers & lt) == 0) hist[warp][l] += __popc(peers);
    __syncwarp();
  }
}

// grid BH, block 256. tiles[h][t] = (group, start, rows, kv_len).
__global__ void tiles_kernel(const int32_t* __restrict__ q_off, const int32_t* __restrict__ k_off,
                             const uint64_t* __restrict__ kmask, int Gq, int Gk, int W, int cap,
                             int block_q, int32_t* __restrict__ tiles,
                             int32_t* __restrict__ tile_count, int ucap, int32_t* __restrict__ units,
                             int32_t* __restrict__ unit_count) {
  __shared__ int nt[kMaxGroups], base[kMaxGroups], kvl[kMaxGroups], nu[kMaxGroups], ubase[kMaxGroups];
  const int h = blockIdx.x, tid = threadIdx.x;
  const int32_t* qo = q_off + static_cast<size_t>(h) * (Gq + 1);
  const int32_t* ko = k_off + static_cast<size_t>(h) * (Gk + 1);
  const uint64_t* km = kmask + static_cast<size_t>(h) * Gq * W;
  for (int g = tid; g < Gq; g += blockDim.x) {
    int n = qo[g + 1] - qo[g];
    nt[g] = (n + block_q - 1) / block_q;
    nu[g] = (n + kUnitRows - 1) / kUnitRows;
    int L = 0;
    for (int b = 0; b < Gk; ++b)
      if ((km[g * W + b / 64] >> (b % 64)) & 1ull) L += ko[b + 1] - ko[b];
    kvl[g] = L;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0, urun = 0;
    for (int g = 0; g < Gq; ++g) {
      base[g] = run;
      run += nt[g];
      ubase[g] = urun;
      urun += nu[g];
    }
    tile_count[h] = min(run, cap);
    unit_count[h] = min(urun, ucap);
  }
  __syncthreads();
  int32_t* th = tiles + static_cast<size_t>(h) * cap * 4;
  for (int g = tid; g < Gq; g += blockDim.x) {
    const int n = qo[g + 1] - qo[g];
    for (int t = 0; t < nt[g]; ++t) {
      const int slot = base[g] + t;
      if (slot >= cap) break;
      th[slot * 4 + 0] = g;
      th[slot * 4 + 1] = qo[g] + t * block_q;
      th[slot * 4 + 2] = min(block_q, n - t * block_q);
      th[slot * 4 + 3] = kvl[g];
    }
    int32_t* uh = units + static_cast<size_t>(h) * ucap * 4;
    for (int u = 0; u < nu[g]; ++u) {
      const int slot = ubase[g] + u;
      if (slot >= ucap) break;
      uh[slot * 4 + 0] = g;
      uh[slot * 4 + 1] = qo[g] + u * kUnitRows;
      uh[slot * 4 + 2] = min(kUnitRows, n - u * kUnitRows);
      uh[slot * 4 + 3] = kvl[g];
    }
  }
}

// dst[h][p] = src[h][perm[h][p]], rows of d bf16. One warp per two rows (d=128)
// or four rows (d=64); grid-stride over BH*N rows.
__global__ void gather_kernel(const uint16_t* __restrict__ src, const int32_t* __restrict__ perm,
                              long long rows_total, int N, int d, uint16_t* __restrict__ dst) {
  const int vec_per_row = d / 8;  // 16-byte vectors
  const long long nvec = rows_total * vec_per_row;
  for (long long e = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; e < nvec;
       e += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = e / vec_per_row;
    const int v = static_cast<int>(e - row * vec_per_row);
    const long long h = row / N;
    int sr = perm[row];
    if (sr < 0 || sr >= N) sr = 0;
    const uint4* s = reinterpret_cast<const uint4*>(src + (h * N + sr) * d) + v;
    reinterpret_cast<uint4*>(dst + row * d)[v] = __ldg(s);
  }
}

}  // namespace svoo

using namespace svoo;

extern "C" svoo_status svoo_permute(const svoo_shape* shape, const void* q, const void* k,
                                    const void* v, const int32_t* k_assign, int n_qc, int n_kc,
                                    int block_q, const svoo_plan* plan, void* qp, void* kp, void* vp,
                                    int32_t* dev_err, void* stream) {
  if (!shape_ok(shape) || !q || !k || !v || !k_assign || !plan || !qp || !kp || !vp)
    return SVOO_ERR_INVALID_ARG;
  if (!plan->kmask || !plan->q_label || !plan->q_perm || !plan->q_off || !plan->k_perm ||
      !plan->k_off || !plan->tiles || !plan->tile_count || !plan->units || !plan->unit_count)
    return SVOO_ERR_INVALID_ARG;
  if (n_qc < 1 || n_qc > 256 || n_kc < 1 || n_kc > 256) return SVOO_ERR_INVALID_ARG;
  if (block_q != 64 && block_q != 128) return SVOO_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(qp, 16) || !aligned(kp, 16) ||
      !aligned(vp, 16))
    return SVOO_ERR_INVALID_ARG;
  const int BH = bh_of(shape), N = shape->N, d = shape->d, nv = nvideo_of(shape);
  const int Gq = groups_q(shape, n_qc), Gk = groups_k(shape, n_kc), W = mask_words(shape, n_kc);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  sort_kernel<<<dim3(BH, 2), kSortWarps * 32, 0, st>>>(plan->q_label, k_assign, N, nv, Gq, Gk, n_kc,
                                                      plan->q_perm, plan->q_off, plan->k_perm,
                                                      plan->k_off, dev_err);
  tiles_kernel<<<BH, 256, 0, st>>>(plan->q_off, plan->k_off, plan->kmask, Gq, Gk, W,
                                   tile_cap(shape, n_qc, block_q), block_q, plan->tiles,
                                   plan->tile_count, unit_cap(shape, n_qc), plan->units,
                                   plan->unit_count);
  const long long rows = static_cast<long long>(BH) * N;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = sms * 8;
  gather_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(q), plan->q_perm, rows, N, d,
                                      static_cast<uint16_t*>(qp));
  gather_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(k), plan->k_perm, rows, N, d,
                                      static_cast<uint16_t*>(kp));
  gather_kernel<<<grid, 256, 0, st>>>(static_cast<const uint16_t*>(v), plan->k_perm, rows, N, d,
                                      static_cast<uint16_t*>(vp));
  return launch_status();
}
