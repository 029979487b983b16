// lr_load.cuh — loads of bf16 row segments whose start is only 2-byte
// aligned (a [K, r] factor with odd r has rows that start anywhere).
//
// Each lane of a group of G lanes loads one 16-byte (or 8-byte) aligned
// chunk, takes the next chunk from its neighbour with a shuffle, and shifts
// the pair so that it ends up with 8 (or 4) consecutive elements of the
// segment.  HBM traffic is the same as for an aligned row: every byte of the
// segment is fetched once; only the chunk that straddles the end of a group
// is fetched by two lanes.  The tensor's own extent [lo, hi) bounds every
// access: chunks that straddle it are read element by element and the part
// outside reads as zero.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

namespace lr {

__device__ __forceinline__ uint4 ld_nc_v4(uintptr_t a) {
  uint4 v;
  asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(a));
  return v;
}

__device__ __forceinline__ uint2 ld_nc_v2(uintptr_t a) {
  uint2 v;
  asm("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(a));
  return v;
}

__device__ __forceinline__ uint32_t ld_u16_or0(uintptr_t p, uintptr_t lo, uintptr_t hi) {
  if (p < lo || p + 2 > hi) return 0u;
  unsigned short h;
  asm("ld.global.nc.u16 %0, [%1];" : "=h"(h) : "l"(p));
  return h;
}

// A chunk that straddles the tensor's first or last byte: element by element
// (rare; kept out of line so that unrolled loops stay small).
static __device__ __noinline__ uint4 chunk16_edge(uintptr_t a, uintptr_t lo, uintptr_t hi) {
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (a + 16 <= lo || a >= hi) return v;
  v.x = ld_u16_or0(a + 0, lo, hi) | (ld_u16_or0(a + 2, lo, hi) << 16);
  v.y = ld_u16_or0(a + 4, lo, hi) | (ld_u16_or0(a + 6, lo, hi) << 16);
  v.z = ld_u16_or0(a + 8, lo, hi) | (ld_u16_or0(a + 10, lo, hi) << 16);
  v.w = ld_u16_or0(a + 12, lo, hi) | (ld_u16_or0(a + 14, lo, hi) << 16);
  return v;
}

// The aligned 16-byte chunk at a, with bytes outside [lo, hi) read as zero.
__device__ __forceinline__ uint4 chunk16(uintptr_t a, uintptr_t lo, uintptr_t hi) {
  if (a >= lo && a + 16 <= hi) return ld_nc_v4(a);
  return chunk16_edge(a, lo, hi);
}

__device__ __forceinline__ uint2 chunk8(uintptr_t a, uintptr_t lo, uintptr_t hi) {
  if (a >= lo && a + 8 <= hi) return ld_nc_v2(a);
  uint2 v = make_uint2(0u, 0u);
  if (a + 8 <= lo || a >= hi) return v;
  v.x = ld_u16_or0(a + 0, lo, hi) | (ld_u16_or0(a + 2, lo, hi) << 16);
  v.y = ld_u16_or0(a + 4, lo, hi) | (ld_u16_or0(a + 6, lo, hi) << 16);
  return v;
}

// High half of x, low half of y: the bf16 pair that starts one element into x.
__device__ __forceinline__ uint32_t mid16(uint32_t x, uint32_t y) {
  return __byte_perm(x, y, 0x5432);
}

// Elements [s, s+8) of the 16-element concatenation (c, n), s in 0..7.
__device__ __forceinline__ uint4 realign16(uint4 c, uint4 n, int s) {
  switch (s) {
    case 0: return c;
    case 1: return make_uint4(mid16(c.x, c.y), mid16(c.y, c.z), mid16(c.z, c.w), mid16(c.w, n.x));
    case 2: return make_uint4(c.y, c.z, c.w, n.x);
    case 3: return make_uint4(mid16(c.y, c.z), mid16(c.z, c.w), mid16(c.w, n.x), mid16(n.x, n.y));
    case 4: return make_uint4(c.z, c.w, n.x, n.y);
    case 5: return make_uint4(mid16(c.z, c.w), mid16(c.w, n.x), mid16(n.x, n.y), mid16(n.y, n.z));
    case 6: return make_uint4(c.w, n.x, n.y, n.z);
    default: return make_uint4(mid16(c.w, n.x), mid16(n.x, n.y), mid16(n.y, n.z), mid16(n.z, n.w));
  }
}

// The same without a branch on s, for groups narrower than a warp whose lanes
// may hold rows with different shifts (a switch would diverge).
__device__ __forceinline__ uint4 realign16_nb(uint4 c, uint4 n, int s) {
  uint32_t w0 = c.x, w1 = c.y, w2 = c.z, w3 = c.w, w4 = n.x, w5 = n.y, w6 = n.z, w7 = n.w;
  if (s & 4) {  // drop two words
    w0 = w2; w1 = w3; w2 = w4; w3 = w5; w4 = w6; w5 = w7;
  }
  if (s & 2) {  // drop one word
    w0 = w1; w1 = w2; w2 = w3; w3 = w4; w4 = w5;
  }
  if (s & 1) {  // drop one element
    return make_uint4(mid16(w0, w1), mid16(w1, w2), mid16(w2, w3), mid16(w3, w4));
  }
  return make_uint4(w0, w1, w2, w3);
}

// Elements [s, s+4) of the 8-element concatenation (c, n), s in 0..3.
__device__ __forceinline__ uint2 realign8(uint2 c, uint2 n, int s) {
  switch (s) {
    case 0: return c;
    case 1: return make_uint2(mid16(c.x, c.y), mid16(c.y, n.x));
    case 2: return make_uint2(c.y, n.x);
    default: return make_uint2(mid16(c.y, n.x), mid16(n.x, n.y));
  }
}

__device__ __forceinline__ uint4 shfl_down_u4(uint4 v, int d, int width) {
  v.x = __shfl_down_sync(0xffffffffu, v.x, d, width);
  v.y = __shfl_down_sync(0xffffffffu, v.y, d, width);
  v.z = __shfl_down_sync(0xffffffffu, v.z, d, width);
  v.w = __shfl_down_sync(0xffffffffu, v.w, d, width);
  return v;
}

__device__ __forceinline__ uint2 shfl_down_u2(uint2 v, int d, int width) {
  v.x = __shfl_down_sync(0xffffffffu, v.x, d, width);
  v.y = __shfl_down_sync(0xffffffffu, v.y, d, width);
  return v;
}

// Bytes [sh, sh + 16) of the 32-byte window (lo, hi), sh even: the 8
// elements that start sh bytes into the aligned granule lo.
__device__ __forceinline__ uint4 window16(const uint4& lo, const uint4& hi, uint32_t sh) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t o[5];
  switch (sh >> 2) {
    case 0: o[0] = w[0]; o[1] = w[1]; o[2] = w[2]; o[3] = w[3]; o[4] = w[4]; break;
    case 1: o[0] = w[1]; o[1] = w[2]; o[2] = w[3]; o[3] = w[4]; o[4] = w[5]; break;
    case 2: o[0] = w[2]; o[1] = w[3]; o[2] = w[4]; o[3] = w[5]; o[4] = w[6]; break;
    default: o[0] = w[3]; o[1] = w[4]; o[2] = w[5]; o[3] = w[6]; o[4] = w[7]; break;
  }
  if (sh & 2u) {
    return make_uint4(__byte_perm(o[0], o[1], 0x5432), __byte_perm(o[1], o[2], 0x5432),
                      __byte_perm(o[2], o[3], 0x5432), __byte_perm(o[3], o[4], 0x5432));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Zero the elements of an 8-element chunk whose index (0..7) is >= keep.
__device__ __forceinline__ uint4 mask_tail8(uint4 v, int keep) {
  if (keep >= 8) return v;
  if (keep <= 0) return make_uint4(0u, 0u, 0u, 0u);
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e0 = 2 * i, e1 = 2 * i + 1;
    uint32_t m = (e0 < keep ? 0x0000FFFFu : 0u) | (e1 < keep ? 0xFFFF0000u : 0u);
    w[i] &= m;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint2 mask_tail4(uint2 v, int keep) {
  if (keep >= 4) return v;
  if (keep <= 0) return make_uint2(0u, 0u);
  uint32_t w[2] = {v.x, v.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int e0 = 2 * i, e1 = 2 * i + 1;
    uint32_t m = (e0 < keep ? 0x0000FFFFu : 0u) | (e1 < keep ? 0xFFFF0000u : 0u);
    w[i] &= m;
  }
  return make_uint2(w[0], w[1]);
}

// Row-segment fetch, split in two so that many loads can be in flight before
// the first one is consumed: seg16_issue() only loads, seg16_finish()
// shuffles and realigns.  A group of G lanes (g = lane index within the
// group, G a power of two dividing 32) fetches the segment that starts at
// element pointer p (2-byte aligned): after finish, lane g holds elements
// [8g, 8g+8) of it, with elements at index >= nvalid set to zero.  All lanes
// of a group share p, hence the shift s = seg_shift(p).
//   cur: aligned chunk g, i.e. segment elements [8g - s, 8g - s + 8)
//   ext: (lane G-1 only) the chunk after the group's last one
__device__ __forceinline__ int seg_shift(const __nv_bfloat16* p) {
  return static_cast<int>((reinterpret_cast<uintptr_t>(p) & 15u) >> 1);
}

__device__ __forceinline__ void seg16_issue(const __nv_bfloat16* p, int g, int G, int nvalid,
                                            uintptr_t lo, uintptr_t hi, uint4& cur, uint4& ext) {
  const uintptr_t a = reinterpret_cast<uintptr_t>(p);
  const uintptr_t base = a & ~static_cast<uintptr_t>(15);
  const int s = static_cast<int>((a & 15u) >> 1);
  // Fast path (the common case, decided once per group): the whole segment is
  // wanted and every chunk the group touches lies inside the tensor.
  if (nvalid >= 8 * G && base >= lo && base + 16u * (G + 1) <= hi) {
    cur = ld_nc_v4(base + 16u * g);
    ext = (g == G - 1 && s != 0) ? ld_nc_v4(base + 16u * G) : make_uint4(0u, 0u, 0u, 0u);
    return;
  }
  const bool need = nvalid > 0 && 8 * g - s < nvalid;
  cur = need ? chunk16(base + 16u * g, lo, hi) : make_uint4(0u, 0u, 0u, 0u);
  ext = (g == G - 1 && s != 0 && 8 * G - s < nvalid) ? chunk16(base + 16u * G, lo, hi)
                                                    : make_uint4(0u, 0u, 0u, 0u);
}

__device__ __forceinline__ uint4 seg16_finish(uint4 cur, uint4 ext, int s, int g, int G,
                                              int nvalid) {
  uint4 nxt = shfl_down_u4(cur, 1, G);
  if (g == G - 1) nxt = ext;
  const uint4 v = (G == 32) ? realign16(cur, nxt, s) : realign16_nb(cur, nxt, s);
  return (nvalid >= 8 * G) ? v : mask_tail8(v, nvalid - 8 * g);
}

}  // namespace lr
