// attn.cu -- block-sparse flash attention over the kept cluster pairs, sm_100a.
//
// One CTA per work unit: up to 256 consecutive rows of one merged query group
// in the cluster-ordered copy qp, as two 128-row query tiles A and B that share
// every key/value tile. The key/value sequence of the group is the
// concatenation, in ascending key-group order, of the kept key groups' rows of
// kp/vp, cut into 16-row chunks (each group's last chunk partly valid, its
// extra rows masked); 8 chunks make one 128-row KV tile. Online (safe) softmax
// runs over those tiles only; O goes back to token order.
//
// Warp roles (384 threads):
//   warp 0      producer: TMA loads of Q_A, Q_B and of every K/V chunk into a
//               2-stage ring (K and V with separate full/empty barriers)
//   warp 1      TMEM owner (512 columns) and, lane 0, the tcgen05 MMA issuer,
//               in the order PV_A(j-1), S_A(j), PV_B(j-1), S_B(j): while one
//               tile's softmax runs, the tensor core works on the other tile
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: thread r owns
//               query row r (= TMEM lane r); reads S_t(j), masks invalid keys,
//               keeps the running max (rescaling O_t in TMEM only when the max
//               grows by more than 2^8) and the sum of the bf16-rounded P,
//               writes P_t(j) as packed bf16 into the upper half of S_t's
//               columns, from where the next MMA reads it as its A operand
//   warps 2-3   idle
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+d), O_B [384,384+d).
// The producer / consumer split follows the flash-attention pipeline that the
// PSA page describes for Hopper (appendix B), rebuilt on tcgen05 + TMEM.
#include "common.cuh"
#include "internal.h"

namespace svoo {

constexpr int kAttnThreads = 384;
constexpr int kQRows = 128;
constexpr int kKvRows = 128;
constexpr int kChunkRows = 16;
constexpr int kChunksPerTile = kKvRows / kChunkRows;
constexpr int kMaxKeyGroups = 264;
constexpr int kTmemCols = 512;
constexpr int kTmemS0 = 0;     // S_A; S_B at +128
constexpr int kTmemO0 = 256;   // O_A; O_B at +128
constexpr int kPOff = 64;      // P_t within S_t's columns (64 packed bf16 pairs)
constexpr float kRescaleLog2 = 8.0f;
constexpr int kRegsLaunch = 168;  // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsLow = 64;      // warps 0-3: TMA producer, MMA issuer
constexpr int kRegsHigh = 216;    // warps 4-11: softmax of the two query tiles
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kAttnThreads * kRegsLaunch, "register split");

struct AttnSmem {
  uint64_t q_full;
  uint64_t k_full[2], v_full[2], k_empty[2], v_empty[2];
  uint64_t s_full[2], p_half[2], p_full[2];
  uint64_t o_done, mma_final;
#ifdef SVOO_TEST_STALL
  uint64_t stall;  // test-only: a barrier that nothing completes
#endif
  uint32_t tmem_base;
  int abort;
  int ncl;      // kept key groups with at least one row
  int nchunks;  // 16-row chunks of the kv sequence
  int cl_row[kMaxKeyGroups];     // first row of the group in kp/vp (global row index)
  int cl_n[kMaxKeyGroups];       // rows of the group
  int cl_c0[kMaxKeyGroups + 1];  // first chunk index of the group
};
constexpr int kAttnHeader = 4096;
static_assert(sizeof(AttnSmem) <= kAttnHeader, "attention header overflow");

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16, A read from tensor memory.
__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// acc + lo + hi of a packed bf16 pair, each widened exactly and added in fp32
// (sm_100 mixed-precision add): the row sum sees the same rounded P that the
// PV product consumes, so the normalisation matches the numerator.
__device__ __forceinline__ float add_bf16x2(uint32_t pk, float acc) {
  float r;
  asm("{\n\t.reg .b16 lo, hi;\n\t.reg .f32 t;\n\t"
      "mov.b32 {lo, hi}, %1;\n\t"
      "add.rn.f32.bf16 t, lo, %2;\n\t"
      "add.rn.f32.bf16 %0, hi, t;\n\t}"
      : "=f"(r)
      : "r"(pk), "f"(acc));
  return r;
}

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
                       const int32_t* __restrict__ k_off, const int32_t* __restrict__ units,
                       const int32_t* __restrict__ unit_count, const int32_t* __restrict__ q_perm,
                       int N, int BH, int Gq, int Gk, int W, int ucap, float scale_log2,
                       uint16_t* __restrict__ out, int* __restrict__ err) {
  constexpr int kSub = D / 64;                // 64-column sub-tiles per row
  constexpr int kTileBytes = kQRows * D * 2;  // one Q, K or V tile
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnSmem* S = reinterpret_cast<AttnSmem*>(base);
  uint8_t* q_s = base + kAttnHeader;       // Q_A, Q_B
  uint8_t* k_s = q_s + 2 * kTileBytes;     // 2 stages
  uint8_t* v_s = k_s + 2 * kTileBytes;     // 2 stages

  const int h = blockIdx.y, x = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (x >= unit_count[h]) return;
  // the error word can change under us: decide once for the whole CTA
  if (__syncthreads_or(timed_out_before(err) ? 1 : 0)) return;
  const int32_t* un = units + (static_cast<size_t>(h) * ucap + x) * 4;
  const int g = un[0], start = un[1], rows = un[2];
  if (g < 0 || g >= Gq || start < 0 || rows < 1 || rows > 2 * kQRows || start + rows > N) {
    if (tid == 0) report_error(err, kErrBadPlan);
    return;
  }
  const bool has_b = rows > kQRows;
  const int rows_t[2] = {min(rows, kQRows), rows - min(rows, kQRows)};

  if (tid == 0) {
    S->abort = 0;
    mbar_init(smem_u32(&S->q_full), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&S->k_full[s]), 1);
      mbar_init(smem_u32(&S->v_full[s]), 1);
      mbar_init(smem_u32(&S->k_empty[s]), 1);
      mbar_init(smem_u32(&S->v_empty[s]), 1);
      mbar_init(smem_u32(&S->s_full[s]), 1);
      mbar_init(smem_u32(&S->p_half[s]), 4);  // one arrival per softmax warp of the tile
      mbar_init(smem_u32(&S->p_full[s]), 4);
    }
    mbar_init(smem_u32(&S->o_done), 1);
    mbar_init(smem_u32(&S->mma_final), 1);
#ifdef SVOO_TEST_STALL
    mbar_init(smem_u32(&S->stall), 1);
#endif
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
      int incl = take ? nchk : 0;  // inclusive scan of the chunk counts of the taken lanes
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
  const uint32_t q_u = smem_u32(q_s), k_u = smem_u32(k_s), v_u = smem_u32(v_s);

  // registers: the producer / issuer warpgroup gives up what the softmax
  // warpgroups use (launch: 384 x 168 = 128 x kRegsLow + 256 x kRegsHigh);
  // each warpgroup's branch starts with its own setmaxnreg
  int k_armed = -1, v_armed = -1;  // producer: last tile whose K / V load was issued
  if (warp < 4) {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
  if (warp == 0 && nkv > 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      mbar_arrive_expect_tx(smem_u32(&S->q_full), (has_b ? 2 : 1) * kTileBytes);
      for (int t = 0; t < (has_b ? 2 : 1); ++t)
        for (int s = 0; s < kSub; ++s)
          tma_load_2d(&qmap, q_u + t * kTileBytes + s * kQRows * 128, smem_u32(&S->q_full), s * 64,
                      h * N + start + t * kQRows);
    }
    ChunkCursor cur;
    const bool issuer = lane < kChunksPerTile * kSub;
    const int my_chunk = lane / kSub, my_sub = lane % kSub;
    auto warp_wait = [&](uint32_t bar, uint32_t parity) -> bool {  // lane 0 waits, the warp follows
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
  } else if (warp == 1 && nkv > 0) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kQRows, kKvRows, false, false);
      const uint32_t idesc_o = idesc_bf16_f32(kQRows, D, false, true);
      const int ntile = has_b ? 2 : 1;
      bool ok = mbar_wait(smem_u32(&S->q_full), 0, abort);
#ifdef SVOO_TEST_STALL
      ok = ok && mbar_wait(smem_u32(&S->stall), 0, abort);  // nothing completes it
#endif
      for (int j = 0; j <= nkv && ok; ++j) {
        const int st = j & 1, pst = (j - 1) & 1;
        for (int t = 0; t < ntile && ok; ++t) {
          if (j >= 1) {  // O_t += P_t(j-1) V_{j-1}, P from TMEM, in two halves of 64 keys
            ok = mbar_wait(smem_u32(&S->p_half[t]), (j - 1) & 1, abort);
            if (ok && t == 0) ok = mbar_wait(smem_u32(&S->v_full[pst]), ((j - 1) >> 1) & 1, abort);
            for (int hf = 0; hf < 2 && ok; ++hf) {
              if (hf == 1) ok = mbar_wait(smem_u32(&S->p_full[t]), (j - 1) & 1, abort);
              if (!ok) break;
              tc_fence_after();
#pragma unroll
              for (int k4 = 0; k4 < kKvRows / 32; ++k4) {
                const int kk = hf * (kKvRows / 32) + k4;
                const uint64_t bd = sw128_desc(v_u + pst * kTileBytes + kk * 16 * 128, kKvRows * 128, 1024);
                umma_f16_ts(tmem + kTmemO0 + t * 128, tmem + kTmemS0 + t * 128 + kPOff + kk * 8, bd, idesc_o,
                            (j > 1 || kk > 0) ? 1u : 0u);
              }
            }
            if (!ok) break;
          }
          if (j < nkv) {  // S_t(j) = Q_t K_j^T; K_j is waited for after PV_A(j-1) is issued,
                          // so a late K tile does not hold back the product that is ready
            if (t == 0) ok = mbar_wait(smem_u32(&S->k_full[st]), (j >> 1) & 1, abort);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t ad = sw128_desc(q_u + t * kTileBytes + (kk >> 2) * kQRows * 128 + (kk & 3) * 32, 16, 1024);
              const uint64_t bd = sw128_desc(k_u + st * kTileBytes + (kk >> 2) * kKvRows * 128 + (kk & 3) * 32, 16, 1024);
              umma_f16(tmem + kTmemS0 + t * 128, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
            }
            umma_commit(smem_u32(&S->s_full[t]));
          }
        }
        if (!ok) break;
        if (j >= 1) umma_commit(smem_u32(&S->v_empty[pst]));
        if (j < nkv) umma_commit(smem_u32(&S->k_empty[st]));
      }
      umma_commit(smem_u32(&S->o_done));
      // every MMA of this thread done before the TMEM is released
      umma_commit(smem_u32(&S->mma_final));
      mbar_wait_cleanup(smem_u32(&S->mma_final), 0);
    }
  }
  } else {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
  if (warp < 8 || has_b) {
    // ---------------------------------------------------------------- softmax of tile t
    const int t = (warp - 4) >> 2;
    const int r = tid - 128 * (1 + t);  // query row within the tile == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t s_col = kTmemS0 + t * 128, o_col = kTmemO0 + t * 128;
    float m = -INFINITY, l = 0.f;
    ChunkCursor cur;
    bool ok = nkv > 0;
    for (int j = 0; j < nkv && ok; ++j) {
      // validity of tile j's chunks, worked out before waiting for S_t(j); it is
      // the same for every row, so the masking branch below is warp-uniform
      int vmask[kChunksPerTile];
      bool full = true;
#pragma unroll
      for (int c8 = 0; c8 < kChunksPerTile; ++c8) {
        int row_unused;
        cur.at(S, j * kChunksPerTile + c8, 0, row_unused, vmask[c8]);
        full = full && vmask[c8] == kChunkRows;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->s_full[t]), j & 1, abort));
      if (!ok) break;
      tc_fence_after();
      float s[kKvRows];
      // all four loads in flight, then one wait that carries the registers
      tmem_ld32f(lane_base + s_col, s);
      tmem_ld32f(lane_base + s_col + 32, s + 32);
      tmem_ld32f(lane_base + s_col + 64, s + 64);
      tmem_ld32f(lane_base + s_col + 96, s + 96);
      tmem_wait_ld_f(s);
      tmem_wait_ld_f(s + 32);
      tmem_wait_ld_f(s + 64);
      tmem_wait_ld_f(s + 96);
      if (!full) {  // a key group's last, partial chunk: invalid keys get -inf (P = 0)
#pragma unroll
        for (int c8 = 0; c8 < kChunksPerTile; ++c8)
#pragma unroll
          for (int c = 0; c < kChunkRows; ++c)
            if (c >= vmask[c8]) s[c8 * kChunkRows + c] = -INFINITY;
      }
      // row max (raw scores; scale_log2 > 0 keeps the order): four chains of
      // three-input maxima
      float m4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int c = 4; c < kKvRows; c += 8) {
        m4[0] = fmax3(m4[0], s[c], s[c + 1]);
        m4[1] = fmax3(m4[1], s[c + 2], s[c + 3]);
        if (c + 4 < kKvRows) {
          m4[2] = fmax3(m4[2], s[c + 4], s[c + 5]);
          m4[3] = fmax3(m4[3], s[c + 6], s[c + 7]);
        }
      }
      const float mx = fmaxf(fmax3(m4[0], m4[1], m4[2]), m4[3]) * scale_log2;
      // running max (log2 units): moved only when it grows by more than 2^8 (P stays <= 2^8)
      const bool grow = mx > m + kRescaleLog2;
      const float alpha = (j > 0 && grow) ? ex2_approx(m - mx) : 1.f;
      if (grow || j == 0) m = fmaxf(m, mx);
      // P = 2^(s scale_log2 - m) (argument by packed fp32 pairs), packed bf16
      // pairs into the upper half of S_t's columns; the first 64 keys are
      // released to the MMA before the rest
      const uint64_t sc2 = f2pack(scale_log2, scale_log2), nm2 = f2pack(-m, -m);
      float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          float x0, x1, p0, p1;
          f2unpack(f2fma(f2pack(s[q * 32 + 2 * c], s[q * 32 + 2 * c + 1]), sc2, nm2), x0, x1);
          p0 = ex2_approx(x0);
          p1 = ex2_approx(x1);
          pk[c] = pack_bf16x2(p0, p1);
          rs8[c & 7] = add_bf16x2(pk[c], rs8[c & 7]);
        }
        tmem_st16(lane_base + s_col + kPOff + q * 16, pk);
        if (q == 1) {
          if (j > 0 && __any_sync(0xffffffffu, grow)) {
            // rescale this warp's rows of O_t before any of P_t(j) is released (the
            // first P half is only stored so far): O_t is stable, since S_t(j)
            // completed after PV_t(j-1) in the MMA order
#pragma unroll
            for (int qo = 0; qo < D / 16; ++qo) {
              uint32_t v[16];
              tmem_ld16(lane_base + o_col + qo * 16, v);
              tmem_wait_ld();
#pragma unroll
              for (int c = 0; c < 16; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * alpha);
              tmem_st16(lane_base + o_col + qo * 16, v);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&S->p_half[t]));
        }
      }
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      l = l * alpha + rs;
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&S->p_full[t]));
    }
    // ---------------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&S->o_done), 0, abort));
    const int rows_me = rows_t[t];
    if (ok) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int tok = r < rows_me ? q_perm[static_cast<size_t>(h) * N + start + t * kQRows + r] : 0;
      uint16_t* orow = out + (static_cast<size_t>(h) * N + tok) * D;
#pragma unroll
      for (int q = 0; q < D / 32; ++q) {
        uint32_t v[32];
        tmem_ld32(lane_base + o_col + q * 32, v);
        tmem_wait_ld();
        if (r < rows_me && tok >= 0 && tok < N) {
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
    } else if (nkv == 0 && r < rows_me) {
      // no kept key rows: the row's output is zero
      const int tok = q_perm[static_cast<size_t>(h) * N + start + t * kQRows + r];
      if (tok >= 0 && tok < N) {
        uint4* orow = reinterpret_cast<uint4*>(out + (static_cast<size_t>(h) * N + tok) * D);
        for (int c = 0; c < D / 8; ++c) orow[c] = make_uint4(0, 0, 0, 0);
      }
    }
  }
  }
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && *abort) {  // every role is done, so the flag is final here
    report_error(err, kErrTimeoutAttn);
    // let every copy the producer issued land before the shared memory goes
    // away (only the last two of each ring can still be in flight)
    if (nkv > 0) {
      for (int j = max(0, k_armed - 1); j <= k_armed; ++j)
        mbar_wait_cleanup(smem_u32(&S->k_full[j & 1]), (j >> 1) & 1);
      for (int j = max(0, v_armed - 1); j <= v_armed; ++j)
        mbar_wait_cleanup(smem_u32(&S->v_full[j & 1]), (j >> 1) & 1);
      mbar_wait_cleanup(smem_u32(&S->q_full), 0);
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
size_t attn_smem_bytes() {
  return 1024 + kAttnHeader + 6 * static_cast<size_t>(kQRows) * D * 2;
}

template <int D>
svoo_status launch_attn(const svoo_shape* sh, const void* qp, const void* kp, const void* vp,
                        const svoo_plan* plan, int n_qc, int n_kc, float scale, void* o,
                        int32_t* dev_err, cudaStream_t st) {
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
  const int ucap = unit_cap(sh, n_qc);
  const float scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  sparse_attn_kernel<D><<<dim3(ucap, BH), kAttnThreads, smem, st>>>(
      qm, km, vm, plan->kmask, plan->k_off, plan->units, plan->unit_count, plan->q_perm, N, BH,
      groups_q(sh, n_qc), groups_k(sh, n_kc), mask_words(sh, n_kc), ucap, scale_log2,
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
  if (!plan->kmask || !plan->k_off || !plan->units || !plan->unit_count || !plan->q_perm)
    return SVOO_ERR_INVALID_ARG;
  if (n_qc < 1 || n_qc > 256 || n_kc < 1 || n_kc > 256) return SVOO_ERR_INVALID_ARG;
  if (block_q != 64 && block_q != 128) return SVOO_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !isfinite(scale)) return SVOO_ERR_INVALID_ARG;
  if (!aligned(qp, 16) || !aligned(kp, 16) || !aligned(vp, 16) || !aligned(o, 16))
    return SVOO_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (shape->d == 128) return launch_attn<128>(shape, qp, kp, vp, plan, n_qc, n_kc, scale, o, dev_err, st);
  return launch_attn<64>(shape, qp, kp, vp, plan, n_qc, n_kc, scale, o, dev_err, st);
}
