// psa.cu -- the static stripe mask of "PSA: Parameterized Stripe Attention"
// (sec. 3.2, Algorithm 1) as a second source of the sparse plan.
//
// Each PSABlock of the (T', H', W') block grid over the video tokens becomes
// one query group and one key group; the mask bit of a block pair is the
// mask definition of Algorithm 1 evaluated on block coordinates (frame index
// a / (H'W'), in-frame index a % (H'W')), since PSA masks at PSABlock
// granularity. The stable sort of svoo_permute then puts every block's tokens
// together in raster order inside the block, which is PSA's block-centric
// (T', H', W', bt, bh, bw) layout, and svoo_sparse_attn runs unchanged. Edge
// blocks keep only their real tokens: the kernels take ragged groups, so the
// paper's 3D padding is not needed.
//
// psa_label_kernel  the block of every token (q_label, and k_assign for the
//                   video tokens); text tokens take group nb.
// psa_mask_kernel   one CTA per block-mask row: the row's bits, the block's size,
//                   and its share of the head's stats.
#include "common.cuh"
#include "internal.h"

namespace svoo {

namespace {

constexpr int kPsaMaxBlocks = 256;

struct PsaGrid {
  int T, H, W;     // video token grid
  int bt, bh, bw;  // PSABlock
  int Tb, Hb, Wb;  // block grid
  int nb;          // Tb * Hb * Wb
};

// grid (ceil(N / 256), BH), block 256
__global__ void __launch_bounds__(256)
    psa_label_kernel(PsaGrid g, int N, int nv, int32_t* __restrict__ q_label,
                     int32_t* __restrict__ k_assign) {
  const int h = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  int a = g.nb;
  if (i < nv) {
    const int hw = g.H * g.W;
    const int t = i / hw, r = i - t * hw;
    const int y = r / g.W, x = r - y * g.W;
    a = ((t / g.bt) * g.Hb + y / g.bh) * g.Wb + x / g.bw;
    k_assign[static_cast<size_t>(h) * nv + i] = a;
  }
  q_label[static_cast<size_t>(h) * N + i] = a;
}

// Algorithm 1 on block indices a (query) and b (key), hw blocks per frame.
__device__ __forceinline__ bool psa_attends(long long a, long long b, long long hw, const long long* p) {
  const long long dt = b / hw - a / hw;
  const long long ra = dt - p[1];
  if ((ra < 0 ? -ra : ra) % p[2] > p[0] - 1) return false;
  const long long ds = b % hw - a % hw;
  const long long rs = ds - p[4];
  return (rs < 0 ? -rs : rs) % p[5] <= p[3] - 1;
}

__device__ __forceinline__ int edge_extent(int n, int blk, int idx) { return min(blk, n - idx * blk); }

// grid (G, BH), block kPsaRowThreads: one CTA per block-mask row a, one thread
// per key group b (bit b of the row); the warps' ballots are the row's 32-bit
// halves. Row a also writes its block size and adds its kept video pairs and
// query tiles to the head's stats (zeroed by the host before the launch).
constexpr int kPsaRowThreads = 320;  // >= 257 groups, whole 64-bit words

__global__ void __launch_bounds__(kPsaRowThreads)
    psa_mask_kernel(PsaGrid g, const int32_t* __restrict__ params, int n_text, int G, int Wd,
                    int block_q, uint64_t* __restrict__ kmask, int32_t* __restrict__ q_sizes,
                    int32_t* __restrict__ stats, int* __restrict__ err) {
  const int a = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  long long prm[6];
#pragma unroll
  for (int i = 0; i < 6; ++i) prm[i] = params[h * 6 + i];
  const bool ok = prm[0] >= 0 && prm[3] >= 0 && prm[2] >= 1 && prm[5] >= 1;
  if (!ok && a == 0 && tid == 0) report_error(err, kErrBadPlan);
  const long long hw = static_cast<long long>(g.Hb) * g.Wb;
  const int b = tid;
  bool keep = false, video = false;
  if (b < G) {
    if (a == g.nb || b == g.nb) {
      keep = true;
    } else {
      keep = ok && psa_attends(a, b, hw, prm);
      video = keep;
    }
  }
  const unsigned bits = __ballot_sync(0xffffffffu, keep);
  const unsigned vbits = __ballot_sync(0xffffffffu, video);
  int32_t* st = stats + static_cast<size_t>(h) * 8;
  if (lane == 0) {
    if (warp < 2 * Wd) reinterpret_cast<uint32_t*>(kmask + (static_cast<size_t>(h) * G + a) * Wd)[warp] = bits;
    if (vbits) atomicAdd(&st[0], __popc(vbits));
  }
  if (tid == 0) {
    int n;
    if (a < g.nb) {
      const int x = a % g.Wb, y = (a / g.Wb) % g.Hb, t = a / (g.Wb * g.Hb);
      n = edge_extent(g.T, g.bt, t) * edge_extent(g.H, g.bh, y) * edge_extent(g.W, g.bw, x);
    } else {
      n = n_text;
    }
    q_sizes[static_cast<size_t>(h) * G + a] = n;
    const int tiles = (n + block_q - 1) / block_q;
    if (tiles) {
      atomicAdd(&st[5], tiles);
      atomicAdd(&st[6], tiles);
    }
    if (a == 0) st[1] = g.nb;
  }
}

}  // namespace

}  // namespace svoo

using namespace svoo;

extern "C" int svoo_psa_block_count(int grid_t, int grid_h, int grid_w, int block_t, int block_h,
                                    int block_w) {
  if (grid_t < 1 || grid_h < 1 || grid_w < 1 || block_t < 1 || block_h < 1 || block_w < 1) return 0;
  const long long n = static_cast<long long>((grid_t + block_t - 1) / block_t) *
                      ((grid_h + block_h - 1) / block_h) * ((grid_w + block_w - 1) / block_w);
  return n > (1 << 30) ? 0 : static_cast<int>(n);
}

extern "C" svoo_status svoo_psa_mask(const svoo_shape* shape, int grid_t, int grid_h, int grid_w,
                                     int block_t, int block_h, int block_w, const int32_t* params,
                                     int block_q, svoo_plan* plan, int32_t* k_assign,
                                     int32_t* dev_err, void* stream) {
  if (!shape_ok(shape) || !params || !plan || !k_assign) return SVOO_ERR_INVALID_ARG;
  if (!plan->kmask || !plan->q_label || !plan->q_sizes || !plan->stats) return SVOO_ERR_INVALID_ARG;
  if (block_q != 64 && block_q != 128) return SVOO_ERR_INVALID_ARG;
  const int nb = svoo_psa_block_count(grid_t, grid_h, grid_w, block_t, block_h, block_w);
  if (nb < 1 || nb > kPsaMaxBlocks) return SVOO_ERR_INVALID_ARG;
  const int nv = nvideo_of(shape);
  if (static_cast<long long>(grid_t) * grid_h * grid_w != nv) return SVOO_ERR_INVALID_ARG;
  PsaGrid g;
  g.T = grid_t;
  g.H = grid_h;
  g.W = grid_w;
  g.bt = block_t;
  g.bh = block_h;
  g.bw = block_w;
  g.Tb = (grid_t + block_t - 1) / block_t;
  g.Hb = (grid_h + block_h - 1) / block_h;
  g.Wb = (grid_w + block_w - 1) / block_w;
  g.nb = nb;
  const int BH = bh_of(shape), N = shape->N;
  const int G = groups_q(shape, nb), Wd = mask_words(shape, nb);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  psa_label_kernel<<<dim3((N + 255) / 256, BH), 256, 0, st>>>(g, N, nv, plan->q_label, k_assign);
  static_assert(kPsaRowThreads >= kPsaMaxBlocks + 1 && kPsaRowThreads % 64 == 0, "one thread per group");
  if (cudaMemsetAsync(plan->stats, 0, sizeof(int32_t) * 8 * static_cast<size_t>(BH), st) != cudaSuccess)
    return SVOO_ERR_CUDA;
  psa_mask_kernel<<<dim3(G, BH), kPsaRowThreads, 0, st>>>(g, params, shape->n_text, G, Wd, block_q,
                                                          plan->kmask, plan->q_sizes, plan->stats,
                                                          dev_err);
  return launch_status();
}
