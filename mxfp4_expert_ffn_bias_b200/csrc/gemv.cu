// Decode path: routed-expert GEMVs on the CUDA cores.
//
// For small token counts each touched expert sees a handful of rows, so the
// layer is a stream of the routed experts' packed weights (ZeroModels GPT-OSS
// docs, "MXFP4 experts": on decode only the routed experts are dequantised).
// Each block owns 64 weight rows of one touched expert; lane pairs own one row
// and split its 32-element MX blocks between them (split-K), loading each
// block's 16 packed bytes with one 16-byte non-coherent vector load. Codes go
// through the hardware FP4 -> f16x2 converter unscaled; products with the f16
// tokens are accumulated in fp32 by mixed-precision FMAs, and each block's
// partial sum is multiplied by its scale 2^(s-127) once. The two lanes of a
// row are then summed with one shuffle.
//
// Tokens are held in f16: each block stages x[t] * 2^-c_t (c_t from the
// router, chosen so max|x_t| * 2^-c_t lies in [2^14, 2^15)), which keeps every
// bf16 input exactly representable except components more than 2^31 below the
// row maximum; the result is multiplied back by 2^c_t. The SwiGLU output is
// bounded by |a| <= 8 * 7 and is stored and reread in f16 unscaled.
#include "common.cuh"
#include "kernels.cuh"
#include "mx_dequant.cuh"

namespace moe {

constexpr int kGemvThreads = 128;  // 4 warps x 16 rows
constexpr int kGemvUnroll = 4;     // MX blocks in flight per lane

size_t gemv_smem_bytes(int C) { return (size_t)kGemvTok * C * sizeof(uint16_t); }

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <bool kGateUp>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(GemvArgs a) {
  extern __shared__ __align__(16) uint16_t xs[];  // f16 [kGemvTok][C]
  const int slotj = blockIdx.y;
  if (slotj >= *a.n_touched) return;
  const int e = a.touched[slotj];
  const int Me = a.counts[e];
  const int row_base = a.offsets[e];
  const int R = a.R, C = a.C, KB = C / 32, KB2 = KB / 2;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int half = lane & 1;
  const int row = blockIdx.x * kGemvRows + warp * 16 + (lane >> 1);
  const uint8_t* wrow = a.blocks + (size_t)(e * (size_t)R + row) * KB * 16;
  const uint8_t* srow = a.scales + (size_t)(e * (size_t)R + row) * KB;

  for (int m0 = 0; m0 < Me; m0 += kGemvTok) {
    const int mc = min(kGemvTok, Me - m0);
    __syncthreads();  // previous pass finished reading xs
    // stage this pass's token rows as f16
    for (int i = tid; i < mc * (C / 8); i += kGemvThreads) {
      const int m = i / (C / 8), c8 = i % (C / 8);
      uint4 v;
      if (kGateUp) {  // tokens in f16, scaled by 2^-c_t
        const int t = a.perm[row_base + m0 + m] / a.k;
        const float sc = exp2_int(-a.xexp[t]);
        const uint4 raw = reinterpret_cast<const uint4*>(a.xin + (size_t)t * C)[c8];
        v.x = pack_f16x2(bf16_bits_to_float(raw.x & 0xFFFF) * sc, bf16_bits_to_float(raw.x >> 16) * sc);
        v.y = pack_f16x2(bf16_bits_to_float(raw.y & 0xFFFF) * sc, bf16_bits_to_float(raw.y >> 16) * sc);
        v.z = pack_f16x2(bf16_bits_to_float(raw.z & 0xFFFF) * sc, bf16_bits_to_float(raw.z >> 16) * sc);
        v.w = pack_f16x2(bf16_bits_to_float(raw.w & 0xFFFF) * sc, bf16_bits_to_float(raw.w >> 16) * sc);
      } else {
        v = reinterpret_cast<const uint4*>(a.xin + (size_t)(row_base + m0 + m) * C)[c8];
      }
      reinterpret_cast<uint4*>(xs + (size_t)m * C)[c8] = v;
    }
    __syncthreads();

    float acc[kGemvTok];
#pragma unroll
    for (int m = 0; m < kGemvTok; ++m) acc[m] = 0.f;

    for (int j0 = 0; j0 < KB2; j0 += kGemvUnroll) {
      uint4 pk[kGemvUnroll];
      uint32_t sb[kGemvUnroll];
#pragma unroll
      for (int u = 0; u < kGemvUnroll; ++u) {
        const int b = 2 * (j0 + u) + half;
        if (j0 + u < KB2) {
          pk[u] = ldg_stream(wrow + (size_t)b * 16);
          sb[u] = srow[b];
        }
      }
#pragma unroll
      for (int u = 0; u < kGemvUnroll; ++u) {
        if (j0 + u < KB2) {
          const int b = 2 * (j0 + u) + half;
          const float scale = __uint_as_float(sb[u] << 23);
          uint32_t hv[16];
          e2m1x8_to_f16x2(pk[u].x, hv[0], hv[1], hv[2], hv[3]);
          e2m1x8_to_f16x2(pk[u].y, hv[4], hv[5], hv[6], hv[7]);
          e2m1x8_to_f16x2(pk[u].z, hv[8], hv[9], hv[10], hv[11]);
          e2m1x8_to_f16x2(pk[u].w, hv[12], hv[13], hv[14], hv[15]);
#pragma unroll
          for (int m = 0; m < kGemvTok; ++m) {
            if (m < mc) {
              const uint4* xv = reinterpret_cast<const uint4*>(xs + (size_t)m * C + b * 32);
              float p0 = 0.f, p1 = 0.f;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const uint4 v = xv[q];
                fma2_f16_f32(p0, p1, hv[4 * q + 0], v.x);
                fma2_f16_f32(p0, p1, hv[4 * q + 1], v.y);
                fma2_f16_f32(p0, p1, hv[4 * q + 2], v.z);
                fma2_f16_f32(p0, p1, hv[4 * q + 3], v.w);
              }
              acc[m] = fmaf(p0 + p1, scale, acc[m]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int m = 0; m < kGemvTok; ++m) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], 1);

    if (kGateUp) {
      // lanes 4i hold gate row 2i, lanes 4i+2 hold up row 2i+1
      float up[kGemvTok];
#pragma unroll
      for (int m = 0; m < kGemvTok; ++m) up[m] = __shfl_down_sync(0xffffffffu, acc[m], 2);
      if ((lane & 3) == 0) {
        const int i = row >> 1;
        const float bg = bf16_bits_to_float(a.bias[(size_t)e * R + row]);
        const float bu = bf16_bits_to_float(a.bias[(size_t)e * R + row + 1]);
        const int I = R / 2;
        for (int m = 0; m < mc; ++m) {
          const int prow = row_base + m0 + m;
          const float sc = exp2_int(a.xexp[a.perm[prow] / a.k]);
          const float g = fminf(acc[m] * sc + bg, 7.f);
          const float uu = fminf(fmaxf(up[m] * sc + bu, -7.f), 7.f);
          const float act = (uu + 1.f) * g * (1.f / (1.f + expf(-1.702f * g)));
          a.act_out[(size_t)prow * I + i] = (uint16_t)(pack_f16x2(act, 0.f) & 0xFFFF);
        }
      }
    } else {
      if (half == 0) {
        const float bd = bf16_bits_to_float(a.bias[(size_t)e * R + row]);
        for (int m = 0; m < mc; ++m) {
          const int p = a.perm[row_base + m0 + m];
          a.slot_out[(size_t)p * R + row] = (acc[m] + bd) * a.wroute[p];
        }
      }
    }
  }
}

// ---------------------------------------------------------------- warp-MMA variant
//
// Same stream and the same numerics (unscaled E2M1 codes -> f16 by the
// hardware converter, f16 tokens, fp32 accumulation, one scale multiply per
// MX block), but the per-block dot products of a warp's 16 rows with up to 8
// tokens run as two m16n8k16 warp MMAs instead of 32 mixed FMAs per token.
// Thread (g = lane/4, q = lane%4) loads word q (bytes 4q..4q+3, elements
// 8q..8q+7) of the MX block of rows g and g+8. The K order inside the MMAs is
// permuted consistently for A and B: MMA 0 takes bytes 4q and 4q+1 as its
// k-slots {2q, 2q+1} and {2q+8, 2q+9}, MMA 1 takes bytes 4q+2 and 4q+3; the
// token fragment of token g is the 16 bytes x[g][32b + 8q .. 32b + 8q + 7].
// Both MMAs of a block cover exactly its 32 elements, so the fp32 result is
// scaled by the row's 2^(s-127) and added to the accumulator.

constexpr int kMmaUnroll = 8;  // MX blocks per pipeline group (two groups in flight)
constexpr int kMmaWarps = 6;   // warps per block (measured best of 4, 6, 8 on the gpt-oss decode shapes)
constexpr int kMmaRows = 16 * kMmaWarps;  // weight rows per block

__device__ __forceinline__ uint32_t ldg_u32(const void* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

__device__ __forceinline__ void mma_16816(float& d0, float& d1, float& d2, float& d3, uint32_t a0, uint32_t a1,
                                          uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1, float c0, float c1,
                                          float c2, float c3) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%10, %11, %12, %13};"
      : "=f"(d0), "=f"(d1), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c0), "f"(c1), "f"(c2), "f"(c3));
}

size_t gemv_mma_smem_bytes(int C) {
  return (size_t)kGemvTok * (C + 8) * sizeof(uint16_t) + (size_t)kMmaRows * (C / 32);
}

struct MmaGroup {
  uint32_t w0[kMmaUnroll], w1[kMmaUnroll];
};

// Loads of MX blocks [b0, b0 + kMmaUnroll) of rows g and g+8 (word q of each
// block); w0p/w1p point at block 0. kFull: every block of the group exists.
template <bool kFull>
__device__ __forceinline__ void mma_load(MmaGroup& G, const uint8_t* w0p, const uint8_t* w1p, int b0, int KB) {
  const uint8_t* p0 = w0p + (size_t)b0 * 16;
  const uint8_t* p1 = w1p + (size_t)b0 * 16;
#pragma unroll
  for (int u = 0; u < kMmaUnroll; ++u) {
    if (kFull || b0 + u < KB) {
      G.w0[u] = ldg_u32(p0 + u * 16);
      G.w1[u] = ldg_u32(p1 + u * 16);
    }
  }
}

// Two m16n8k16 MMAs per MX block, scaled by the rows' 2^(s-127) into acc.
template <bool kFull>
__device__ __forceinline__ void mma_compute(const MmaGroup& G, int b0, int KB, bool has_tok, const uint16_t* xg,
                                            const uint8_t* s0p, const uint8_t* s1p, float& acc0, float& acc1,
                                            float& acc2, float& acc3) {
  const uint16_t* xb = xg + b0 * 32;
  const uint8_t* s0 = s0p + b0;
  const uint8_t* s1 = s1p + b0;
#pragma unroll
  for (int u = 0; u < kMmaUnroll; ++u) {
    if (kFull || b0 + u < KB) {
      uint32_t f0, f1, f2, f3, f4, f5, f6, f7;
      e2m1x8_to_f16x2(G.w0[u], f0, f1, f2, f3);
      e2m1x8_to_f16x2(G.w1[u], f4, f5, f6, f7);
      uint4 xv = make_uint4(0, 0, 0, 0);
      if (has_tok) xv = *reinterpret_cast<const uint4*>(xb + u * 32);
      float d0, d1, d2, d3;
      mma_16816(d0, d1, d2, d3, f0, f4, f1, f5, xv.x, xv.y, 0.f, 0.f, 0.f, 0.f);
      mma_16816(d0, d1, d2, d3, f2, f6, f3, f7, xv.z, xv.w, d0, d1, d2, d3);
      const float sa = __uint_as_float((uint32_t)s0[u] << 23);
      const float sb = __uint_as_float((uint32_t)s1[u] << 23);
      acc0 = fmaf(d0, sa, acc0);
      acc1 = fmaf(d1, sa, acc1);
      acc2 = fmaf(d2, sb, acc2);
      acc3 = fmaf(d3, sb, acc3);
    }
  }
}

// One block = kMmaWarps warps = 16 * kMmaWarps weight rows of one touched
// expert (rows past R idle). Shared memory holds the pass's tokens in f16
// (8 x C, rows padded by 16 bytes) and the block's scale bytes.
template <bool kGateUp>
__global__ void __launch_bounds__(kMmaWarps * 32) gemv_mma_kernel(GemvArgs a) {
  extern __shared__ __align__(16) uint8_t gsm[];
  const int slotj = blockIdx.y;
  if (slotj >= *a.n_touched) return;
  const int e = a.touched[slotj];
  const int Me = a.counts[e];
  const int row_base = a.offsets[e];
  const int R = a.R, C = a.C, KB = C / 32, CP = C + 8;
  uint16_t* xs = reinterpret_cast<uint16_t*>(gsm);                // f16 [8][CP]
  uint8_t* scs = gsm + (size_t)kGemvTok * CP * sizeof(uint16_t);  // [kMmaRows][KB]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int r0 = blockIdx.x * kMmaRows;
  const int rows_here = min(kMmaRows, R - r0);  // a multiple of 16
  const bool warp_on = warp * 16 < rows_here;
  const int rg = r0 + warp * 16 + g;  // this thread's rows rg and rg + 8
  const uint8_t* w0p = a.blocks + ((size_t)e * R + rg) * KB * 16 + q * 4;
  const uint8_t* w1p = w0p + (size_t)8 * KB * 16;
  const uint8_t* s0p = scs + (warp * 16 + g) * KB;
  const uint8_t* s1p = s0p + 8 * KB;
  const int KBfull = KB - KB % (2 * kMmaUnroll);  // blocks covered by full ping-pong rounds
  {
    const uint4* src = reinterpret_cast<const uint4*>(a.scales + ((size_t)e * R + r0) * KB);
    uint4* dst = reinterpret_cast<uint4*>(scs);
    for (int i = tid; i < rows_here * KB / 16; i += kMmaWarps * 32) dst[i] = src[i];
  }

  for (int m0 = 0; m0 < Me; m0 += kGemvTok) {
    const int mc = min(kGemvTok, Me - m0);
    MmaGroup A, B;
    if (warp_on) {  // weights do not depend on the tokens: start loading before staging them
      if (KBfull > 0) mma_load<true>(A, w0p, w1p, 0, KB);
      else mma_load<false>(A, w0p, w1p, 0, KB);
    }
    __syncthreads();
    for (int i = tid; i < mc * (C / 8); i += kMmaWarps * 32) {
      const int m = i / (C / 8), c8 = i % (C / 8);
      uint4 v;
      if (kGateUp) {  // tokens in f16, scaled by 2^-c_t
        const int t = a.perm[row_base + m0 + m] / a.k;
        const float sc = exp2_int(-a.xexp[t]);
        const uint4 raw = reinterpret_cast<const uint4*>(a.xin + (size_t)t * C)[c8];
        v.x = pack_f16x2(bf16_bits_to_float(raw.x & 0xFFFF) * sc, bf16_bits_to_float(raw.x >> 16) * sc);
        v.y = pack_f16x2(bf16_bits_to_float(raw.y & 0xFFFF) * sc, bf16_bits_to_float(raw.y >> 16) * sc);
        v.z = pack_f16x2(bf16_bits_to_float(raw.z & 0xFFFF) * sc, bf16_bits_to_float(raw.z >> 16) * sc);
        v.w = pack_f16x2(bf16_bits_to_float(raw.w & 0xFFFF) * sc, bf16_bits_to_float(raw.w >> 16) * sc);
      } else {
        v = reinterpret_cast<const uint4*>(a.xin + (size_t)(row_base + m0 + m) * C)[c8];
      }
      reinterpret_cast<uint4*>(xs + (size_t)m * CP)[c8] = v;
    }
    __syncthreads();
    if (!warp_on) continue;
    const bool has_tok = g < mc;
    const uint16_t* xg = xs + (size_t)g * CP + 8 * q;
    float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f, acc3 = 0.f;
    int b0 = 0;
    for (; b0 < KBfull; b0 += 2 * kMmaUnroll) {
      mma_load<true>(B, w0p, w1p, b0 + kMmaUnroll, KB);
      mma_compute<true>(A, b0, KB, has_tok, xg, s0p, s1p, acc0, acc1, acc2, acc3);
      if (b0 + 2 * kMmaUnroll < KBfull) mma_load<true>(A, w0p, w1p, b0 + 2 * kMmaUnroll, KB);
      else mma_load<false>(A, w0p, w1p, b0 + 2 * kMmaUnroll, KB);
      mma_compute<true>(B, b0 + kMmaUnroll, KB, has_tok, xg, s0p, s1p, acc0, acc1, acc2, acc3);
    }
    if (b0 < KB) {  // tail: fewer than 2 * kMmaUnroll blocks, group A already loaded
      mma_load<false>(B, w0p, w1p, b0 + kMmaUnroll, KB);
      mma_compute<false>(A, b0, KB, has_tok, xg, s0p, s1p, acc0, acc1, acc2, acc3);
      mma_compute<false>(B, b0 + kMmaUnroll, KB, has_tok, xg, s0p, s1p, acc0, acc1, acc2, acc3);
    }
    // acc0/acc1: row rg, tokens 2q, 2q+1; acc2/acc3: row rg+8, same tokens
    const int n0 = 2 * q, n1 = 2 * q + 1;
    if (kGateUp) {
      const float u0 = __shfl_down_sync(0xffffffffu, acc0, 4), u1 = __shfl_down_sync(0xffffffffu, acc1, 4);
      const float u2 = __shfl_down_sync(0xffffffffu, acc2, 4), u3 = __shfl_down_sync(0xffffffffu, acc3, 4);
      if ((g & 1) == 0) {
        const int I = R / 2;
        for (int h2 = 0; h2 < 2; ++h2) {
          const int row = rg + 8 * h2;  // even: gate row; row + 1: up row
          const float bg = bf16_bits_to_float(a.bias[(size_t)e * R + row]);
          const float bu = bf16_bits_to_float(a.bias[(size_t)e * R + row + 1]);
          for (int jj = 0; jj < 2; ++jj) {
            const int n = jj ? n1 : n0;
            if (n >= mc) continue;
            const float gacc = h2 ? (jj ? acc3 : acc2) : (jj ? acc1 : acc0);
            const float uacc = h2 ? (jj ? u3 : u2) : (jj ? u1 : u0);
            const int prow = row_base + m0 + n;
            const float sc = exp2_int(a.xexp[a.perm[prow] / a.k]);
            const float gg = fminf(gacc * sc + bg, 7.f);
            const float uu = fminf(fmaxf(uacc * sc + bu, -7.f), 7.f);
            const float act = (uu + 1.f) * gg * (1.f / (1.f + expf(-1.702f * gg)));
            a.act_out[(size_t)prow * I + (row >> 1)] = (uint16_t)(pack_f16x2(act, 0.f) & 0xFFFF);
          }
        }
      }
    } else {
      for (int h2 = 0; h2 < 2; ++h2) {
        const int row = rg + 8 * h2;
        const float bd = bf16_bits_to_float(a.bias[(size_t)e * R + row]);
        for (int jj = 0; jj < 2; ++jj) {
          const int n = jj ? n1 : n0;
          if (n >= mc) continue;
          const float v = h2 ? (jj ? acc3 : acc2) : (jj ? acc1 : acc0);
          const int p = a.perm[row_base + m0 + n];
          a.slot_out[(size_t)p * R + row] = (v + bd) * a.wroute[p];
        }
      }
    }
  }
}

cudaError_t configure_gemv(int Cmax) {
  const size_t smem = gemv_smem_bytes(Cmax);
  const size_t smem_mma = gemv_mma_smem_bytes(Cmax);
  cudaError_t err = raise_smem_limit((const void*)gemv_kernel<true>, smem);
  if (err == cudaSuccess) err = raise_smem_limit((const void*)gemv_kernel<false>, smem);
  if (err == cudaSuccess) err = raise_smem_limit((const void*)gemv_mma_kernel<true>, smem_mma);
  if (err == cudaSuccess) err = raise_smem_limit((const void*)gemv_mma_kernel<false>, smem_mma);
  return err;
}

cudaError_t launch_gemv_gateup(const GemvArgs& a, int max_touched, int variant, int sm_count, cudaStream_t st) {
  (void)sm_count;
  if (variant == 1) {
    dim3 grid((a.R + kMmaRows - 1) / kMmaRows, max_touched);
    gemv_mma_kernel<true><<<grid, kMmaWarps * 32, gemv_mma_smem_bytes(a.C), st>>>(a);
  } else {
    dim3 grid(a.R / kGemvRows, max_touched);
    gemv_kernel<true><<<grid, kGemvThreads, gemv_smem_bytes(a.C), st>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemv_down(const GemvArgs& a, int max_touched, int variant, int sm_count, cudaStream_t st) {
  (void)sm_count;
  if (variant == 1) {
    dim3 grid((a.R + kMmaRows - 1) / kMmaRows, max_touched);
    gemv_mma_kernel<false><<<grid, kMmaWarps * 32, gemv_mma_smem_bytes(a.C), st>>>(a);
  } else {
    dim3 grid(a.R / kGemvRows, max_touched);
    gemv_kernel<false><<<grid, kGemvThreads, gemv_smem_bytes(a.C), st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace moe
