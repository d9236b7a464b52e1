// internal.h -- host-side helpers shared by the library's translation units:
// argument checks, workspace carving, tensor-map encoding and launch checks.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/svoo.h"

namespace svoo {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline bool shape_ok(const svoo_shape* s) {
  if (!s) return false;
  if (s->B < 1 || s->H < 1 || s->n_text < 0) return false;
  if (s->d != 64 && s->d != 128) return false;
  if (s->N - s->n_text < 1 || s->N > (1 << 20)) return false;
  if (static_cast<long long>(s->B) * s->H > 65535) return false;  // grid.y limit
  // TMA row coordinates are int32: keep every row of [B*H*N, d] addressable
  if (static_cast<long long>(s->B) * s->H * s->N >= (1LL << 31) - 256) return false;
  return true;
}

inline int bh_of(const svoo_shape* s) { return s->B * s->H; }
inline int nvideo_of(const svoo_shape* s) { return s->N - s->n_text; }
inline int groups_q(const svoo_shape* s, int n_qc) { return n_qc + (s->n_text > 0 ? 1 : 0); }
inline int groups_k(const svoo_shape* s, int n_kc) { return n_kc + (s->n_text > 0 ? 1 : 0); }
inline int mask_words(const svoo_shape* s, int n_kc) { return (groups_k(s, n_kc) + 63) / 64; }
inline int tile_cap(const svoo_shape* s, int n_qc, int block_q) {
  return (s->N + block_q - 1) / block_q + groups_q(s, n_qc);
}
// cluster count padded for the scoring MMA: a multiple of 64, since two
// threads share a score row and each reads its half from TMEM 32 columns at a time
// attention work units: up to 256 rows of one query group
constexpr int kUnitRows = 256;
inline int unit_cap(const svoo_shape* s, int n_qc) {
  return (s->N + kUnitRows - 1) / kUnitRows + groups_q(s, n_qc);
}
inline int pad64(int c) { return (c + 63) / 64 * 64; }

// Bump allocator over a caller-provided workspace (256-byte aligned pieces).
struct Carver {
  char* base;
  size_t used = 0;
  explicit Carver(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t count) {
    used = (used + 255) / 256 * 256;
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
};

// cuTensorMapEncodeTiled, fetched once through the runtime (no -lcuda needed).
CUresult encode_tiled_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                         uint32_t box_rows, uint32_t box_cols);

inline svoo_status launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SVOO_OK : SVOO_ERR_CUDA;
}

}  // namespace svoo
