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

}  // namespace moe
