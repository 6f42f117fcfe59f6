// Pieces shared by the 1-CTA and 2-CTA grouped GEMM kernels: parameters,
// tile decoding over the device-side expert offsets, and the fused epilogues.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace moe {

struct GemmParams {
  int E;
  int K;        // reduction length
  int n_out;    // output row length: I (mlp1) or D (mlp2)
  int n_tile;   // output columns per tile
  int mma_n;    // MMA N: 2*n_tile (mlp1) or n_tile (mlp2)
  int NT;       // column tiles per expert
  int b_rows;   // rows of B per expert: 2I (mlp1) or D (mlp2)
  int64_t R;
  const int32_t* offsets;
  const uint16_t* bias;
  const int32_t* perm;
  const float* topk_w;
  void* out;  // h (R, I) bf16 for mlp1; o_perm (R, D) fp32 for mlp2
  int* status;
  Act act;    // mlp1's activation
};

// Tile `tile` -> (expert e, column tile nt, row tile mt) for row tiles of bm
// rows; tpre[e] = first tile of expert e (tiles numbered expert-major).
__device__ __forceinline__ void decode_tile(int tile, const int* tpre, const int* seg, int E, int bm, int& e,
                                            int& nt, int& mt) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (tpre[mid] <= tile)
      lo = mid;
    else
      hi = mid - 1;
  }
  e = lo;
  const int local = tile - tpre[e];
  const int mtiles = (seg[e + 1] - seg[e] + bm - 1) / bm;
  nt = local / mtiles;
  mt = local - nt * mtiles;
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
  }
}

// Fused epilogue of one accumulator tile for the thread's row: bias + SwiGLU
// (or its GPT-OSS variant)
// into h (bf16), or bias times the gate weight into o (fp32). tbase is the
// TMEM address of the thread's lane at column 0 of the accumulator; row is
// the routed row, valid = row inside the expert segment.
template <bool kSwiGLU>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, uint32_t tbase, int e, int nt, int64_t row,
                                              bool valid) {
  using namespace sm100;
  // Columns are drained 32 at a time: up to four 8-column TMEM loads per
  // wait (the bounds are warp-uniform, as tcgen05.ld requires).
  if (kSwiGLU) {
    const uint16_t* bg = p.bias + static_cast<int64_t>(e) * p.b_rows + nt * p.n_tile;
    const uint16_t* bu = bg + p.n_out;
    uint16_t* dst = static_cast<uint16_t*>(p.out) + row * p.n_out + nt * p.n_tile;
    for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
      uint32_t g[32], u[32];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (c0 + 8 * j < p.n_tile) {
          tmem_ld_x8(tbase + c0 + 8 * j, g + 8 * j);
          tmem_ld_x8(tbase + p.n_tile + c0 + 8 * j, u + 8 * j);
        }
      }
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + 8 * j;
        if (c < p.n_tile) {
          float gb[8], ub[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(bg + c)), gb);
          unpack8(__ldg(reinterpret_cast<const uint4*>(bu + c)), ub);
          float hv[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float gate = __uint_as_float(g[8 * j + i]) + gb[i];
            const float up = __uint_as_float(u[8 * j + i]) + ub[i];
            hv[i] = glu_act(gate, up, p.act);
          }
          if (valid) {
            uint4 v;
            v.x = pack_bf16x2(hv[0], hv[1]);
            v.y = pack_bf16x2(hv[2], hv[3]);
            v.z = pack_bf16x2(hv[4], hv[5]);
            v.w = pack_bf16x2(hv[6], hv[7]);
            *reinterpret_cast<uint4*>(dst + c) = v;
          }
        }
      }
    }
  } else {
    float wgt = 0.f;
    if (valid) {
      const int32_t a = p.perm[row];
      if (a >= 0 && a < p.R)
        wgt = p.topk_w[a];
      else
        record_status(p.status, MOE_ERR_DEVICE_BOUNDS);
    }
    const uint16_t* bb = p.bias + static_cast<int64_t>(e) * p.b_rows + nt * p.n_tile;
    float* dst = static_cast<float*>(p.out) + row * p.n_out + nt * p.n_tile;
    for (int c0 = 0; c0 < p.n_tile; c0 += 32) {
      uint32_t v[32];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (c0 + 8 * j < p.n_tile) tmem_ld_x8(tbase + c0 + 8 * j, v + 8 * j);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int c = c0 + 8 * j;
        if (c < p.n_tile) {
          float bv[8];
          unpack8(__ldg(reinterpret_cast<const uint4*>(bb + c)), bv);
          float ov[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) ov[i] = wgt * (__uint_as_float(v[8 * j + i]) + bv[i]);
          // one 32-byte store: a full sector per thread (rows are 32-byte aligned)
          if (valid) st_global_v8f(dst + c, ov);
        }
      }
    }
  }
}

}  // namespace moe
