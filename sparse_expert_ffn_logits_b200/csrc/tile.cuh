// tile.cuh - the two warp-level contractions of the layer, for 16 weight rows x 8 tokens.
//
// tile_dot:  D[r][c] = sum_h W[row r][h] * x[token c][h]           (router, gate, up)
// tile_down: Y[h][c] += sum_r W_down^T[row r][h] * hc[r][c]          (down, 64 h per call)
//
// Thread (g = lane/4, t = lane%4) of a warp holds the mma.m16n8k16 accumulator fragment
//   d0 = D[g][2t], d1 = D[g][2t+1], d2 = D[g+8][2t], d3 = D[g+8][2t+1]
// in both the bf16 (tensor-core) and the fp32 (CUDA-core) variants, so the epilogues are shared.
//
// bf16 tile_dot reads each weight row with 16-byte loads: thread t of a row takes h = 32b + 8t
// .. +8 of block b and uses them as the k-slots {2t, 2t+1, 2t+8, 2t+9} of two consecutive mmas.
// The same permutation of the contraction index is applied to the token operand, so the sum is
// unchanged while every load stays a full 16-byte vector.
//
// bf16 tile_down has the neuron index as the contraction index and reads 16-byte vectors of
// four rows (2t, 2t+1, 2t+8, 2t+9) at h0 + 8g; a byte permute pairs the same h of two rows into
// one A register.  Output row m of m-tile i is h = h0 + 8g + 2i (m = g) or h0 + 8g + 2i + 1
// (m = g + 8): the output index is permuted instead of the loads.
#pragma once

#include "common.cuh"

namespace moe {

template <int UNROLL>
__device__ __forceinline__ void tile_dot(const __nv_bfloat16* rowA, const __nv_bfloat16* rowB,
                                         const __nv_bfloat16* const* xtok, int b0, int bstep,
                                         int nblk, float d[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const __nv_bfloat16* xg = xtok[g];
  for (int b = b0; b < nblk; b += bstep * UNROLL) {
    uint4 wa[UNROLL], wb[UNROLL], xv[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int bb = b + u * bstep;
      if (bb < nblk) {
        const int off = bb * 32 + t * 8;
        wa[u] = ld_stream(rowA + off);
        wb[u] = ld_stream(rowB + off);
        xv[u] = xg ? ld_nc(xg + off) : make_uint4(0, 0, 0, 0);
      } else {
        wa[u] = wb[u] = xv[u] = make_uint4(0, 0, 0, 0);
      }
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      mma_16816(d, wa[u].x, wb[u].x, wa[u].y, wb[u].y, xv[u].x, xv[u].y);
      mma_16816(d, wa[u].z, wb[u].z, wa[u].w, wb[u].w, xv[u].z, xv[u].w);
    }
  }
}

template <int UNROLL>
__device__ __forceinline__ void tile_dot(const float* rowA, const float* rowB,
                                         const float* const* xtok, int b0, int bstep, int nblk,
                                         float d[4]) {
  const int lane = threadIdx.x & 31, t = lane & 3;
  const float* x0 = xtok[2 * t];
  const float* x1 = xtok[2 * t + 1];
  for (int b = b0; b < nblk; b += bstep) {
#pragma unroll 2
    for (int v = 0; v < 8; ++v) {
      const int off = b * 32 + v * 4;
      const float4 a = *reinterpret_cast<const float4*>(rowA + off);
      const float4 c = *reinterpret_cast<const float4*>(rowB + off);
      const float4 y0 = x0 ? *reinterpret_cast<const float4*>(x0 + off) : make_float4(0, 0, 0, 0);
      const float4 y1 = x1 ? *reinterpret_cast<const float4*>(x1 + off) : make_float4(0, 0, 0, 0);
      d[0] += a.x * y0.x + a.y * y0.y + a.z * y0.z + a.w * y0.w;
      d[1] += a.x * y1.x + a.y * y1.y + a.z * y1.z + a.w * y1.w;
      d[2] += c.x * y0.x + c.y * y0.y + c.z * y0.z + c.w * y0.w;
      d[3] += c.x * y1.x + c.y * y1.y + c.z * y1.z + c.w * y1.w;
    }
  }
}

// bf16 down: drow[r] = start of row r's down half; hc words: b0 = rows (2t, 2t+1) of token g,
// b1 = rows (2t+8, 2t+9) of token g.
__device__ __forceinline__ void tile_down(const __nv_bfloat16* const* drow, int h0, uint32_t b0,
                                          uint32_t b1, const void* /*unused*/, float acc[4][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int off = h0 + 8 * g;
  const uint4 r0 = ld_stream(drow[2 * t] + off);
  const uint4 r1 = ld_stream(drow[2 * t + 1] + off);
  const uint4 r2 = ld_stream(drow[2 * t + 8] + off);
  const uint4 r3 = ld_stream(drow[2 * t + 9] + off);
  const uint32_t w0[4] = {r0.x, r0.y, r0.z, r0.w};
  const uint32_t w1[4] = {r1.x, r1.y, r1.z, r1.w};
  const uint32_t w2[4] = {r2.x, r2.y, r2.z, r2.w};
  const uint32_t w3[4] = {r3.x, r3.y, r3.z, r3.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t a0 = __byte_perm(w0[i], w1[i], 0x5410);
    const uint32_t a1 = __byte_perm(w0[i], w1[i], 0x7632);
    const uint32_t a2 = __byte_perm(w2[i], w3[i], 0x5410);
    const uint32_t a3 = __byte_perm(w2[i], w3[i], 0x7632);
    mma_16816(acc[i], a0, a1, a2, a3, b0, b1);
  }
}

// fp32 down: hcf = [16 rows][8 tokens] floats in shared memory.
__device__ __forceinline__ void tile_down(const float* const* drow, int h0, uint32_t, uint32_t,
                                          const void* hcf_v, float acc[4][4]) {
  const float(*hcf)[8] = reinterpret_cast<const float(*)[8]>(hcf_v);
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int off = h0 + 8 * g;
#pragma unroll 4
  for (int r = 0; r < 16; ++r) {
    const float4 lo = *reinterpret_cast<const float4*>(drow[r] + off);
    const float4 hi = *reinterpret_cast<const float4*>(drow[r] + off + 4);
    const float v[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
    const float c0 = hcf[r][2 * t], c1 = hcf[r][2 * t + 1];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[i][0] += v[2 * i] * c0;
      acc[i][1] += v[2 * i] * c1;
      acc[i][2] += v[2 * i + 1] * c0;
      acc[i][3] += v[2 * i + 1] * c1;
    }
  }
}

// Sums the kWarps partial fragments (red[w][lane][4]) into warp 0's d; the caller syncs before.
__device__ __forceinline__ void reduce_fragments(const float (*red)[32][4], float d[4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w][lane][c];
    d[c] = s;
  }
}

}  // namespace moe
