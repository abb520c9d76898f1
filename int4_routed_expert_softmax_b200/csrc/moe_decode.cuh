// moe_decode.cuh -- device pieces of the decode (GEMV) expert kernels shared by
// the three-kernel decode path (moe_decode.cu) and the fused batch-1 kernel
// (moe_fused.cu): one lane's chunk of an int4 gs64 row against a Q8_0 vector
// (dp4a on the offset-binary nibbles, exact integer block sums, fp32 scales in
// the kernels' fixed order), the loads of a row chunk and of an activation
// chunk, and the left-to-right sum of a row's 32 chunk values.
#pragma once

#include "moe_device.cuh"

namespace moe {

__host__ __device__ inline size_t al128d(size_t v) { return (v + 127) / 128 * 128; }

// ---------------------------------------------------------------------------
// Integer + fp32 dot of one lane's chunk of a weight row with one activation
// vector.  w: packed words of the chunk's groups, act: 16 words per group
// (elements 64g .. 64g+63), d: the two block scales per group, z: the integer
// start values per group, -8 * (code sum of block 2g) and -128 * (code sum of
// block 2g+1), which turn the unsigned nibble sums into exact signed sums.
// ---------------------------------------------------------------------------
template <int CSZ>
__device__ __forceinline__ float chunk_dot(const uint32_t (&w)[CSZ][8], const float (&sc)[CSZ],
                                           const uint32_t (&act)[CSZ][16], const float (&d)[CSZ][2],
                                           const int (&z)[CSZ][2], int c0, int G) {
  float acc = 0.0f;
#pragma unroll
  for (int gi = 0; gi < CSZ; ++gi) {
    if (c0 + gi < G) {
      int s0 = z[gi][0], s1 = z[gi][1], t0 = 0, t1 = 0;  // two chains per block
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s0 = dp4a_us(w[gi][j] & 0x0F0F0F0Fu, act[gi][j], s0);
        t0 = dp4a_us(w[gi][4 + j] & 0x0F0F0F0Fu, act[gi][4 + j], t0);
        s1 = dp4a_us(w[gi][j] & 0xF0F0F0F0u, act[gi][8 + j], s1);
        t1 = dp4a_us(w[gi][4 + j] & 0xF0F0F0F0u, act[gi][12 + j], t1);
      }
      s0 += t0;  // sum (u - 8) q over the low nibbles (block 2g)
      s1 += t1;  // 16 * sum (u - 8) q over the high nibbles (block 2g+1)
      const float fa = fmul((float)s0, d[gi][0]);
      const float fb = ffma(fmul((float)s1, 0.0625f), d[gi][1], fa);  // (float)s1/16 is exact
      acc = ffma(sc[gi], fb, acc);
    }
  }
  return acc;
}

// Sum of the first nch of 32 chunk values, left to right (fixed order).
__device__ __forceinline__ float chunk_sum(const float *rr, int nch) {
  float v[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) v[c] = (c < nch) ? rr[c] : 0.0f;
  float tot = v[0];
#pragma unroll
  for (int c = 1; c < 32; ++c)
    if (c < nch) tot = fadd(tot, v[c]);
  return tot;
}

// Weight words and scales of one row's chunk (CSZ groups) from shared memory.
template <int CSZ>
__device__ __forceinline__ void load_row(const unsigned char *rowp, const __half *scp, int c0, int G,
                                         uint32_t (&w)[CSZ][8], float (&sc)[CSZ]) {
#pragma unroll
  for (int gi = 0; gi < CSZ; ++gi) {
    const int g = c0 + gi;
    if (g < G) {
      const uint4 w0 = *reinterpret_cast<const uint4 *>(rowp + 32 * g);
      const uint4 w1 = *reinterpret_cast<const uint4 *>(rowp + 32 * g + 16);
      w[gi][0] = w0.x;
      w[gi][1] = w0.y;
      w[gi][2] = w0.z;
      w[gi][3] = w0.w;
      w[gi][4] = w1.x;
      w[gi][5] = w1.y;
      w[gi][6] = w1.z;
      w[gi][7] = w1.w;
      sc[gi] = __half2float(scp[g]);
    } else {
#pragma unroll
      for (int z = 0; z < 8; ++z) w[gi][z] = 0u;
      sc[gi] = 0.0f;
    }
  }
}

// Activation chunk (CSZ groups) of one token: 16 words, 2 scales and the two
// integer start values per group.
template <int CSZ>
__device__ __forceinline__ void load_act(const unsigned char *xa, const float *xd, const int *qs,
                                         int c0, int G, uint32_t (&act)[CSZ][16], float (&d)[CSZ][2],
                                         int (&z)[CSZ][2]) {
#pragma unroll
  for (int gi = 0; gi < CSZ; ++gi) {
    const int g = c0 + gi;
    const uint4 *src = reinterpret_cast<const uint4 *>(xa + 64 * gi);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 v = g < G ? src[q] : make_uint4(0u, 0u, 0u, 0u);  // no read past the vector's groups
      act[gi][4 * q] = v.x;
      act[gi][4 * q + 1] = v.y;
      act[gi][4 * q + 2] = v.z;
      act[gi][4 * q + 3] = v.w;
    }
    d[gi][0] = g < G ? xd[2 * g] : 0.0f;
    d[gi][1] = g < G ? xd[2 * g + 1] : 0.0f;
    z[gi][0] = g < G ? -8 * qs[2 * g] : 0;
    z[gi][1] = g < G ? -128 * qs[2 * g + 1] : 0;
  }
}

// ---------------------------------------------------------------------------
// MXFP4 rows (32 E2M1 codes per E8M0 exponent; two consecutive elements per
// byte, the lower-indexed one in the low nibble; one exponent byte per
// 32-block after the row's codes).  Twice an E2M1 value is an integer in
// [-12, 12], so a block's products with Q8_0 codes sum exactly in int32:
// S_b = sum 2 e2m1 q; the block term is (S_b d_b) 2^(E_b - 128).
// ---------------------------------------------------------------------------

// Four E2M1 codes (the four nibbles of x, element i in bits 4i..4i+3) as four
// signed bytes 2 * e2m1: magnitudes and negated magnitudes by byte permutes of
// constant tables indexed by the low three bits, then per byte the one the
// sign bit selects.
__device__ __forceinline__ uint32_t e2m1x4_to_s8(uint32_t x) {
  const uint32_t sel = x & 0x7777u;
  const uint32_t pos = __byte_perm(0x03020100u, 0x0C080604u, sel);  // 0 1 2 3 | 4 6 8 12
  const uint32_t neg = __byte_perm(0xFDFEFF00u, 0xF4F8FAFCu, sel);  // their negatives
  return __byte_perm(pos, neg, 0x3210u | ((x >> 1) & 0x4444u));
}

// 2^k as a float for -149 <= k <= 127 (exact: a normal or subnormal power of two).
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __int_as_float((k + 127) << 23) : __int_as_float(1 << (k + 149));
}

// Codes and exponent pairs of one row's chunk (CSZ 64-element groups).
template <int CSZ>
__device__ __forceinline__ void load_row_mx(const unsigned char *rowp, const unsigned char *exps, int c0, int G,
                                            uint32_t (&w)[CSZ][8], uint32_t (&ex)[CSZ]) {
#pragma unroll
  for (int gi = 0; gi < CSZ; ++gi) {
    const int g = c0 + gi;
    if (g < G) {
      const uint4 w0 = *reinterpret_cast<const uint4 *>(rowp + 32 * g);
      const uint4 w1 = *reinterpret_cast<const uint4 *>(rowp + 32 * g + 16);
      w[gi][0] = w0.x;
      w[gi][1] = w0.y;
      w[gi][2] = w0.z;
      w[gi][3] = w0.w;
      w[gi][4] = w1.x;
      w[gi][5] = w1.y;
      w[gi][6] = w1.z;
      w[gi][7] = w1.w;
      ex[gi] = *reinterpret_cast<const uint16_t *>(exps + 2 * g);  // blocks 2g, 2g+1
    } else {
#pragma unroll
      for (int z = 0; z < 8; ++z) w[gi][z] = 0u;
      ex[gi] = 0u;
    }
  }
}

// The lane's chunk of an MXFP4 row against one Q8_0 vector (act, d as for
// chunk_dot): per block, S_b by dp4a of the decoded codes with the codes of x,
// then acc += (S_b d_b) 2^(E_b - 128), blocks in ascending order.
template <int CSZ>
__device__ __forceinline__ float chunk_dot_mx(const uint32_t (&w)[CSZ][8], const uint32_t (&ex)[CSZ],
                                              const uint32_t (&act)[CSZ][16], const float (&d)[CSZ][2], int c0,
                                              int G) {
  float acc = 0.0f;
#pragma unroll
  for (int gi = 0; gi < CSZ; ++gi) {
    if (c0 + gi < G) {
      int s0 = 0, s1 = 0, t0 = 0, t1 = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {  // word j: elements 8j .. 8j+7 of the block
        s0 = __dp4a((int)e2m1x4_to_s8(w[gi][j] & 0xFFFFu), (int)act[gi][2 * j], s0);
        t0 = __dp4a((int)e2m1x4_to_s8(w[gi][j] >> 16), (int)act[gi][2 * j + 1], t0);
        s1 = __dp4a((int)e2m1x4_to_s8(w[gi][4 + j] & 0xFFFFu), (int)act[gi][8 + 2 * j], s1);
        t1 = __dp4a((int)e2m1x4_to_s8(w[gi][4 + j] >> 16), (int)act[gi][8 + 2 * j + 1], t1);
      }
      const int e0 = (int)(ex[gi] & 0xFFu), e1 = (int)(ex[gi] >> 8);
      acc = fadd(acc, fmul(fmul((float)(s0 + t0), d[gi][0]), pow2f(e0 - 128)));
      acc = fadd(acc, fmul(fmul((float)(s1 + t1), d[gi][1]), pow2f(e1 - 128)));
    }
  }
  return acc;
}

}  // namespace moe
