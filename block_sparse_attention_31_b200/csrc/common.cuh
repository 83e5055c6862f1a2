// common.cuh -- grid geometry shared by the kernels of libvsa: how a head's layout maps
// natural tokens to slots and back, and which key slots of a block are real tokens.
//
// Layouts ("Sparse Video-Gen" summary page, "Approach": temporal heads are re-laid out
// from token-major to frame-major order; "USV" page, Figure 2: local 3D cubes):
//   natural token  t = f*S + s, s = h*Wl + w, S = Hl*Wl, N = F*S
//   spatial head   slot = t
//   temporal head  slot = s*F + f                       (frame-major)
//   cube head      slot = cube*V + ((f%cf)*ch + h%ch)*cw + w%cw,
//                  cube = ((f/cf)*nch + h/ch)*ncw + w/cw, V = cf*ch*cw, padded slots empty
#pragma once
#include <stdint.h>

namespace vsa {

enum : int { kSpatial = 0, kTemporal = 1, kCube = 2 };

struct Geom {
  int F, Hl, Wl, S, N;   // grid
  int cf, ch, cw, vol;   // cube dims (vol = cf*ch*cw), 0 when cubes are unused
  int ncf, nch, ncw;     // cubes per dimension
  int ncubes;            // ncf*nch*ncw
  int R;                 // rows per head of a permuted buffer (N, or ncubes*vol)
  int block;             // tokens per block
  int nblk;              // blocks per head in mask arrays: ceil(R / block)
};

// Rows of a head's buffer in its own layout.
__host__ __device__ __forceinline__ int layout_rows(const Geom& g, int kind) {
  return kind == kCube ? g.ncubes * g.vol : g.N;
}

// Slot of natural token t under `kind`.
__host__ __device__ __forceinline__ int slot_of_token(const Geom& g, int kind, int t) {
  if (kind == kSpatial) return t;
  const int f = t / g.S, s = t - f * g.S;
  if (kind == kTemporal) return s * g.F + f;
  const int h = s / g.Wl, w = s - h * g.Wl;
  const int cube = ((f / g.cf) * g.nch + h / g.ch) * g.ncw + w / g.cw;
  return cube * g.vol + ((f % g.cf) * g.ch + h % g.ch) * g.cw + w % g.cw;
}

// Natural token at `slot` under `kind`, or -1 for a slot that holds no token.
__host__ __device__ __forceinline__ int token_of_slot(const Geom& g, int kind, int slot) {
  if (kind == kSpatial) return slot < g.N ? slot : -1;
  if (kind == kTemporal) {
    if (slot >= g.N) return -1;
    const int s = slot / g.F, f = slot - s * g.F;
    return f * g.S + s;
  }
  const int cube = slot / g.vol, r = slot - cube * g.vol;
  if (cube >= g.ncubes) return -1;
  const int cw_i = cube % g.ncw, ch_i = (cube / g.ncw) % g.nch, cf_i = cube / (g.ncw * g.nch);
  const int dw = r % g.cw, dh = (r / g.cw) % g.ch, df = r / (g.cw * g.ch);
  const int f = cf_i * g.cf + df, h = ch_i * g.ch + dh, w = cw_i * g.cw + dw;
  if (f >= g.F || h >= g.Hl || w >= g.Wl) return -1;
  return (f * g.Hl + h) * g.Wl + w;
}

// Number of real tokens in cube `cube`.
__host__ __device__ __forceinline__ int cube_tokens(const Geom& g, int cube) {
  const int cw_i = cube % g.ncw, ch_i = (cube / g.ncw) % g.nch, cf_i = cube / (g.ncw * g.nch);
  const int nf = min(g.cf, g.F - cf_i * g.cf), nh = min(g.ch, g.Hl - ch_i * g.ch), nw = min(g.cw, g.Wl - cw_i * g.cw);
  return nf * nh * nw;
}

// Whether every slot of key block `kb` under `kind` is a real token.
__host__ __device__ __forceinline__ bool block_full(const Geom& g, int kind, int kb) {
  if (kind != kCube) return (kb + 1) * g.block <= g.N;
  return cube_tokens(g, kb) == g.vol;
}

}  // namespace vsa
