// attn.cu -- block-sparse flash attention over the kept cluster pairs, sm_100a.
//
// One CTA per query tile (<= 128 rows of one merged query group, contiguous in
// the cluster-ordered copy qp). Its key/value sequence is the concatenation,
// in ascending key-group order, of the kept key groups' rows of kp/vp; the
// sequence is cut into 16-row chunks (the last chunk of each group partly
// valid, its extra rows masked) and 8 chunks make one 128-row KV tile. Online
// (safe) softmax runs over those tiles only; O is written in token order.
//
// Warp roles (256 threads):
//   warp 0     producer: TMA loads of the Q tile and of every K/V chunk into a
//              2-stage ring (K and V with separate full/empty barriers)
//   warp 1     TMEM allocation (512 columns) and, lane 0, the tcgen05 MMA
//              issuer: S_j = Q K_j^T into one of two TMEM S buffers, then
//              O += P_{j-1} V_{j-1} into the TMEM O accumulator
//   warps 4-7  softmax: thread r owns query row r (= TMEM lane r); reads S_j,
//              masks invalid key rows, updates the running max / sum, rescales
//              O in TMEM when the max grows, writes P_j (bf16, 128B-swizzled
//              K-major) to shared memory; finally O / l to global memory
//   warps 2-3  idle
// The design follows the producer / consumer flash-attention pipeline that the
// PSA page describes for Hopper (appendix B), rebuilt on tcgen05 + TMEM.
#include "common.cuh"
#include "internal.h"

namespace svoo {

constexpr int kAttnThreads = 256;
constexpr int kQRows = 128;
constexpr int kKvRows = 128;
constexpr int kChunkRows = 16;
constexpr int kChunksPerTile = kKvRows / kChunkRows;
constexpr int kMaxKeyGroups = 264;
constexpr int kTmemCols = 512;
constexpr int kTmemO = 256;

struct AttnSmem {
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], k_empty[2], v_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, pv_done, mma_final;
  uint32_t tmem_base;
  int abort;
  int ncl;      // kept key groups with at least one row
  int nchunks;  // 16-row chunks of the kv sequence
  int cl_row[kMaxKeyGroups];  // first row of the group in kp/vp (global row index)
  int cl_n[kMaxKeyGroups];    // rows of the group
  int cl_c0[kMaxKeyGroups + 1];  // first chunk index of the group
};
constexpr int kAttnHeader = 4096;
static_assert(sizeof(AttnSmem) <= kAttnHeader, "attention header overflow");

// Walks the chunk sequence in increasing order: group of chunk gc, its first
// global row and its valid rows (0 past the end).
struct ChunkCursor {
  int ci = 0;
  __device__ __forceinline__ void at(const AttnSmem* S, int gc, int oob_row, int& row, int& valid) {
    if (gc >= S->nchunks) {
      row = oob_row;
      valid = 0;
      return;
    }
    while (gc >= S->cl_c0[ci + 1]) ++ci;
    const int l = gc - S->cl_c0[ci];
    row = S->cl_row[ci] + l * kChunkRows;
    valid = min(kChunkRows, S->cl_n[ci] - l * kChunkRows);
  }
};

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap qmap,
                       const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, const uint64_t* __restrict__ kmask,
                       const int32_t* __restrict__ k_off, const int32_t* __restrict__ tiles,
                       const int32_t* __restrict__ tile_count, const int32_t* __restrict__ q_perm,
                       int N, int BH, int Gq, int Gk, int W, int cap, float scale_log2,
                       uint16_t* __restrict__ out, int* __restrict__ err) {
  constexpr int kSub = D / 64;                 // 64-column sub-tiles per row
  constexpr int kTileBytes = kQRows * D * 2;   // Q, K or V tile
  constexpr int kPBytes = kQRows * kKvRows * 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnSmem* S = reinterpret_cast<AttnSmem*>(base);
  uint8_t* q_s = base + kAttnHeader;
  uint8_t* k_s = q_s + kTileBytes;         // 2 stages
  uint8_t* v_s = k_s + 2 * kTileBytes;     // 2 stages
  uint8_t* p_s = v_s + 2 * kTileBytes;

  const int h = blockIdx.y, x = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (x >= tile_count[h] || timed_out_before(err)) return;
  const int32_t* tl = tiles + (static_cast<size_t>(h) * cap + x) * 4;
  const int g = tl[0], start = tl[1], rows = tl[2];
  if (g < 0 || g >= Gq || start < 0 || rows < 1 || rows > kQRows || start + rows > N) {
    if (tid == 0) report_error(err, kErrBadPlan);
    return;
  }

  if (tid == 0) {
    S->abort = 0;
    mbar_init(smem_u32(&S->q_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&S->k_full[s]), 1);
      mbar_init(smem_u32(&S->v_full[s]), 1);
      mbar_init(smem_u32(&S->k_empty[s]), 1);
      mbar_init(smem_u32(&S->v_empty[s]), 1);
      mbar_init(smem_u32(&S->s_full[s]), 1);
      mbar_init(smem_u32(&S->s_free[s]), 128);
    }
    mbar_init(smem_u32(&S->p_full), 128);
    mbar_init(smem_u32(&S->pv_done), 1);
    mbar_init(smem_u32(&S->mma_final), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    // kept key groups of query group g, ascending, with their rows in kp/vp
    const int32_t* ko = k_off + static_cast<size_t>(h) * (Gk + 1);
    const uint64_t* km = kmask + (static_cast<size_t>(h) * Gq + g) * W;
    int n_cl = 0, n_ch = 0;
    bool bad = false;
    for (int b0 = 0; b0 < Gk; b0 += 32) {
      const int b = b0 + lane;
      bool take = false;
      int o0 = 0, nb = 0;
      if (b < Gk) {
        o0 = ko[b];
        nb = ko[b + 1] - o0;
        if (o0 < 0 || nb < 0 || o0 + nb > N) bad = true;
        take = ((km[b >> 6] >> (b & 63)) & 1ull) && nb > 0 && !bad;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, take);
      const int pos = n_cl + __popc(bal & ((1u << lane) - 1u));
      const int nchk = (nb + kChunkRows - 1) / kChunkRows;
      // chunk offsets need an exclusive scan of nchk over the taken lanes
      int incl = take ? nchk : 0;
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (take) {
        S->cl_row[pos] = h * N + o0;
        S->cl_n[pos] = nb;
        S->cl_c0[pos] = n_ch + incl - nchk;
      }
      n_cl += __popc(bal);
      n_ch += __shfl_sync(0xffffffffu, incl, 31);
    }
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) {
      S->ncl = n_cl;
      S->nchunks = n_ch;
      S->cl_c0[n_cl] = n_ch;
      if (bad) {
        report_error(err, kErrBadPlan);
        S->ncl = 0;
        S->nchunks = 0;
        S->cl_c0[0] = 0;
      }
    }
  } else if (warp == 1) {
    __syncwarp();
    tmem_alloc(smem_u32(&S->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = S->tmem_base;
  volatile int* abort = &S->abort;
  const int nkv = (S->nchunks + kChunksPerTile - 1) / kChunksPerTile;
  const int oob_row = BH * N;  // past the tensor: TMA fills zeros
  const uint32_t q_u = smem_u32(q_s), k_u = smem_u32(k_s), v_u = smem_u32(v_s), p_u = smem_u32(p_s);

  if (warp == 0 && nkv > 0) {
    // ---------------------------------------------------------------- producer
    int k_armed = -1, v_armed = -1;  // last tile whose K / V load was issued
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      mbar_arrive_expect_tx(smem_u32(&S->q_full), kTileBytes);
      for (int s = 0; s < kSub; ++s)
        tma_load_2d(&qmap, q_u + s * kQRows * 128, smem_u32(&S->q_full), s * 64, h * N + start);
    }
    ChunkCursor cur;
    const bool issuer = lane < kChunksPerTile * kSub;
    const int my_chunk = lane / kSub, my_sub = lane % kSub;
    // lane 0 waits, the warp follows its verdict (keeps the warp converged)
    auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {
      int okl = 1;
      if (lane == 0) okl = mbar_wait(bar, parity, abort) ? 1 : 0;
      return __shfl_sync(0xffffffffu, okl, 0) != 0;
    };
    for (int j = 0; j < nkv; ++j) {
      const int st = j & 1;
      int row = 0, valid = 0;
      if (issuer) cur.at(S, j * kChunksPerTile + my_chunk, oob_row, row, valid);
      if (j >= 2 && !warp_wait(smem_u32(&S->k_empty[st]), ((j - 2) >> 1) & 1)) break;
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(&S->k_full[st]), kTileBytes);
      __syncwarp();
      if (issuer)
        tma_load_2d(&kmap, k_u + st * kTileBytes + my_sub * kKvRows * 128 + my_chunk * kChunkRows * 128,
                    smem_u32(&S->k_full[st]), my_sub * 64, row);
      k_armed = j;
      if (j >= 2 && !warp_wait(smem_u32(&S->v_empty[st]), ((j - 2) >> 1) & 1)) break;
      if (lane == 0) mbar_arrive_expect_tx(smem_u32(&S->v_full[st]), kTileBytes);
      __syncwarp();
      if (issuer)
        tma_load_2d(&vmap, v_u + st * kTileBytes + my_sub * kKvRows * 128 + my_chunk * kChunkRows * 128,
                    smem_u32(&S->v_full[st]), my_sub * 64, row);
      v_armed = j;
    }
    if (*abort && lane == 0) {
      // let every issued copy land before this CTA's shared memory is released
      int dummy = 0;
      for (int j = max(0, k_armed - 1); j <= k_armed; ++j)
        mbar_wait(smem_u32(&S->k_full[j & 1]), (j >> 1) & 1, &dummy);
      for (int j = max(0, v_armed - 1); j <= v_armed; ++j)
        mbar_wait(smem_u32(&S->v_full[j & 1]), (j >> 1) & 1, &dummy);
      dummy = 0;
      mbar_wait(smem_u32(&S->q_full), 0, &dummy);
    }
  } else if (warp == 1 && nkv > 0) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kQRows, kKvRows, false, false);
      const uint32_t idesc_o = idesc_bf16_f32(kQRows, D, false, true);
      bool ok = mbar_wait(smem_u32(&S->q_full), 0, abort);
      auto issue_pv = [&](int jj) -> bool {
        const int st = jj & 1;
        if (!mbar_wait(smem_u32(&S->p_full), jj & 1, abort)) return false;
        if (!mbar_wait(smem_u32(&S->v_full[st]), (jj >> 1) & 1, abort)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kKvRows / 16; ++kk) {
          const uint64_t ad = sw128_desc(p_u + (kk >> 2) * kQRows * 128 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(v_u + st * kTileBytes + kk * 16 * 128, kKvRows * 128, 1024);
          umma_f16(tmem + kTmemO, ad, bd, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(smem_u32(&S->pv_done));
        umma_commit(smem_u32(&S->v_empty[st]));
        return true;
      };
      for (int j = 0; j < nkv && ok; ++j) {
        const int st = j & 1;
        ok = mbar_wait(smem_u32(&S->k_full[st]), (j >> 1) & 1, abort);
        if (ok && j >= 2) ok = mbar_wait(smem_u32(&S->s_free[st]), ((j - 2) >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t ad = sw128_desc(q_u + (kk >> 2) * kQRows * 128 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(k_u + st * kTileBytes + (kk >> 2) * kKvRows * 128 + (kk & 3) * 32, 16, 1024);
          umma_f16(tmem + st * kKvRows, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(smem_u32(&S->s_full[st]));
        umma_commit(smem_u32(&S->k_empty[st]));
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok) issue_pv(nkv - 1);
      // every MMA of this thread done before the TMEM is released
      umma_commit(smem_u32(&S->mma_final));
      int dummy = 0;
      mbar_wait(smem_u32(&S->mma_final), 0, &dummy);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    const int r = tid - 128;  // query row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    float m = -INFINITY, l = 0.f;
    ChunkCursor cur;
    bool ok = true;
    for (int j = 0; j < nkv && ok; ++j) {
      const int st = j & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->s_full[st]), (j >> 1) & 1, abort));
      if (!ok) break;
      tc_fence_after();
      float s[kKvRows];
#pragma unroll
      for (int q = 0; q < kKvRows / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(lane_base + st * kKvRows + q * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 32; ++c) s[q * 32 + c] = __uint_as_float(v[c]);
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&S->s_free[st]));
      float mx = -INFINITY;
#pragma unroll
      for (int c8 = 0; c8 < kChunksPerTile; ++c8) {
        int row_unused, valid;
        cur.at(S, j * kChunksPerTile + c8, 0, row_unused, valid);
#pragma unroll
        for (int c = 0; c < kChunkRows; ++c) {
          const int col = c8 * kChunkRows + c;
          s[col] = c < valid ? s[col] * scale_log2 : -INFINITY;
          mx = fmaxf(mx, s[col]);
        }
      }
      const float m_new = fmaxf(m, mx);
      // a row that has seen no valid key yet keeps m = -inf; use 0 as its
      // reference so that no (-inf) - (-inf) appears
      const float m_ref = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = ex2_approx(m - m_ref);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kKvRows; ++c) {
        s[c] = ex2_approx(s[c] - m_ref);
        rs += s[c];
      }
      l = l * alpha + rs;
      m = m_new;
      if (j >= 1) {
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->pv_done), (j - 1) & 1, abort));
        if (!ok) break;
        tc_fence_after();
        // rescale O when this warp's running max moved (warp-uniform decision,
        // since tcgen05.ld/st are warp-collective)
        if (__any_sync(0xffffffffu, alpha < 1.f)) {
#pragma unroll
          for (int q = 0; q < D / 32; ++q) {
            uint32_t v[32];
            tmem_ld32(lane_base + kTmemO + q * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * alpha);
            tmem_st32(lane_base + kTmemO + q * 32, v);
          }
          tmem_wait_st();
        }
      }
      // P row -> shared memory, 128B-swizzled K-major (two 64-column sub-tiles)
#pragma unroll
      for (int k16 = 0; k16 < kKvRows / 8; ++k16) {
        const int sub = k16 >> 3, kc = k16 & 7;
        uint4 pk;
        pk.x = pack_bf16x2(s[k16 * 8 + 0], s[k16 * 8 + 1]);
        pk.y = pack_bf16x2(s[k16 * 8 + 2], s[k16 * 8 + 3]);
        pk.z = pack_bf16x2(s[k16 * 8 + 4], s[k16 * 8 + 5]);
        pk.w = pack_bf16x2(s[k16 * 8 + 6], s[k16 * 8 + 7]);
        *reinterpret_cast<uint4*>(p_s + sub * kQRows * 128 + r * 128 + ((kc ^ (r & 7)) << 4)) = pk;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&S->p_full));
    }
    // ---------------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->pv_done), (nkv - 1) & 1, abort));
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int tok = r < rows ? q_perm[static_cast<size_t>(h) * N + start + r] : 0;
      uint16_t* orow = out + (static_cast<size_t>(h) * N + tok) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(lane_base + kTmemO + q * 32, v);
        tmem_wait_ld();
        if (r < rows && tok >= 0 && tok < N) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(v[c8 * 8 + 0]) * inv, __uint_as_float(v[c8 * 8 + 1]) * inv);
            pk.y = pack_bf16x2(__uint_as_float(v[c8 * 8 + 2]) * inv, __uint_as_float(v[c8 * 8 + 3]) * inv);
            pk.z = pack_bf16x2(__uint_as_float(v[c8 * 8 + 4]) * inv, __uint_as_float(v[c8 * 8 + 5]) * inv);
            pk.w = pack_bf16x2(__uint_as_float(v[c8 * 8 + 6]) * inv, __uint_as_float(v[c8 * 8 + 7]) * inv);
            reinterpret_cast<uint4*>(orow + q * 32)[c8] = pk;
          }
        }
      }
    }
  }
  if (warp >= 4 && nkv == 0) {
    // no kept key rows: the row's output is zero
    const int r = tid - 128;
    if (r < rows) {
      const int tok = q_perm[static_cast<size_t>(h) * N + start + r];
      if (tok >= 0 && tok < N) {
        uint4 z = make_uint4(0, 0, 0, 0);
        uint4* orow = reinterpret_cast<uint4*>(out + (static_cast<size_t>(h) * N + tok) * D);
        for (int c = 0; c < D / 8; ++c) orow[c] = z;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort) report_error(err, kErrTimeoutAttn);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
size_t attn_smem_bytes() {
  return 1024 + kAttnHeader + 5 * static_cast<size_t>(kQRows) * D * 2 +
         static_cast<size_t>(kQRows) * kKvRows * 2;
}

template <int D>
svoo_status launch_attn(const svoo_shape* sh, const void* qp, const void* kp, const void* vp,
                        const svoo_plan* plan, int n_qc, int n_kc, int block_q, float scale,
                        void* o, int32_t* dev_err, cudaStream_t st) {
  const int BH = bh_of(sh), N = sh->N;
  const uint64_t rows = static_cast<uint64_t>(BH) * N;
  CUtensorMap qm, km, vm;
  if (encode_tiled_2d(&qm, qp, rows, D, kQRows, 64) != CUDA_SUCCESS ||
      encode_tiled_2d(&km, kp, rows, D, kChunkRows, 64) != CUDA_SUCCESS ||
      encode_tiled_2d(&vm, vp, rows, D, kChunkRows, 64) != CUDA_SUCCESS)
    return SVOO_ERR_CUDA;
  const size_t smem = attn_smem_bytes<D>();
  if (cudaFuncSetAttribute(sparse_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess)
    return SVOO_ERR_CUDA;
  const int cap = tile_cap(sh, n_qc, block_q);
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  sparse_attn_kernel<D><<<dim3(cap, BH), kAttnThreads, smem, st>>>(
      qm, km, vm, plan->kmask, plan->k_off, plan->tiles, plan->tile_count, plan->q_perm, N, BH,
      groups_q(sh, n_qc), groups_k(sh, n_kc), mask_words(sh, n_kc), cap, scale_log2,
      static_cast<uint16_t*>(o), dev_err);
  return launch_status();
}

}  // namespace svoo

using namespace svoo;

extern "C" svoo_status svoo_sparse_attn(const svoo_shape* shape, const void* qp, const void* kp,
                                        const void* vp, const svoo_plan* plan, int n_qc, int n_kc,
                                        int block_q, float scale, void* o, int32_t* dev_err,
                                        void* stream) {
  if (!shape_ok(shape) || !qp || !kp || !vp || !plan || !o) return SVOO_ERR_INVALID_ARG;
  if (!plan->kmask || !plan->k_off || !plan->tiles || !plan->tile_count || !plan->q_perm)
    return SVOO_ERR_INVALID_ARG;
  if (n_qc < 1 || n_qc > 256 || n_kc < 1 || n_kc > 256) return SVOO_ERR_INVALID_ARG;
  if (block_q != 64 && block_q != 128) return SVOO_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return SVOO_ERR_INVALID_ARG;
  if (!aligned(qp, 16) || !aligned(kp, 16) || !aligned(vp, 16) || !aligned(o, 16))
    return SVOO_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (shape->d == 128) return launch_attn<128>(shape, qp, kp, vp, plan, n_qc, n_kc, block_q, scale, o, dev_err, st);
  return launch_attn<64>(shape, qp, kp, vp, plan, n_qc, n_kc, block_q, scale, o, dev_err, st);
}
