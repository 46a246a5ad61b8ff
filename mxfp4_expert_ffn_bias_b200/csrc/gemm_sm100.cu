// Prefill path: grouped MXFP4 GEMMs on the 5th-generation tensor cores.
//
// D[rows of expert e, n] = A[rows, K] . dequant(W[e])[n, K]^T, for every
// expert with routed rows, in one persistent launch. A is the bf16 token
// matrix in permuted (expert-grouped) order: the gathered x for gate_up and
// the SwiGLU output for down. W is an MXFP4 tensor (E2M1 codes two per byte,
// one E8M0 scale per 32 K elements; ZeroModels GPT-OSS docs, "MXFP4 experts").
//
// Per CTA (one per SM), warp-specialised:
//   warp 4      TMA producer: A tile (128 x 64 bf16, 128B swizzle) and the
//               packed weight tile (BN x 32 bytes) per K step into a ring of
//               STAGES stages; the tile's E8M0 scales (BN x K/32 bytes,
//               contiguous in memory) with one bulk copy per output tile.
//   warps 6-9   dequantise the packed tile exactly to bf16 (mx_dequant8_bf16)
//               into the stage's B tile, in the same 128B-swizzled K-major
//               layout TMA gives A.
//   warp 5      one thread issues tcgen05.mma kind::f16 (bf16 x bf16 -> fp32,
//               M=128, N=BN, K=16) into a TMEM accumulator; commits free the
//               stage and, at the end of a tile, hand the accumulator over.
//   warps 0-3   epilogue: tcgen05.ld the accumulator (warp w reads TMEM lanes
//               32w..32w+31 = tile rows), add the bias and either
//                 gate_up: de-interleave (even columns = gate, odd = up; MaxText
//                 PR 2647 "1 Support many-to-one transform"), apply the clamped
//                 SwiGLU and store bf16 act[row, n/2], or
//                 down: scale by the routing weight and store fp32 rows of the
//                 slot buffer at the row's (token, slot) pair index.
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile overlap
// the main loop of the next. Every wait is bounded; a wait that gives up sets
// the status word and the CTA winds down.
#include <cstdio>

#include "common.cuh"
#include "kernels.cuh"
#include "mx_dequant.cuh"

namespace moe {

namespace {

constexpr int kThreads = 320;
constexpr int kEpiWarp0 = 0, kProdWarp = 4, kMmaWarp = 5, kDeqWarp0 = 6;
constexpr int kMaxE = 256;

template <int BN, int STAGES>
struct Smem {
  static constexpr int kA = kBM * 128;  // bytes of one A stage
  static constexpr int kB = BN * 128;   // bytes of one dequantised B stage
  static constexpr int kP = BN * 32;    // bytes of one packed stage
  static constexpr int offA = 0;
  static constexpr int offB = offA + STAGES * kA;
  static constexpr int offP = offB + STAGES * kB;
  static constexpr int offSC = offP + STAGES * kP;  // 2 scale buffers of BN*KB bytes (runtime size)
};

struct __align__(8) Bars {
  uint64_t full_ab[8];
  uint64_t full_b[8];
  uint64_t empty[8];
  uint64_t sc_full[2];
  uint64_t sc_empty[2];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int counts[kMaxE];
  int offsets[kMaxE + 1];
  int mt_off[kMaxE + 1];
};

// Dynamic shared memory of one CTA. At least 116 KB, so that no two CTAs of
// this kernel share an SM (each allocates all 512 TMEM columns).
template <int BN, int STAGES>
size_t smem_total(int K) {
  const size_t need = 1024 + Smem<BN, STAGES>::offSC + 2 * (size_t)BN * (K / 32) + sizeof(Bars) + 64;
  return need < 116 * 1024 ? 116 * 1024 : need;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded, abortable wait used by every role: gives up after `limit_us`
// microseconds of wall time (or as soon as another role gave up), raising the
// status word and the CTA's abort flag.
// With abortable = false (used to drain copies and MMAs still in flight before
// the CTA exits) only the time limit ends the wait.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, long long limit_us, volatile int* abort_flag,
                                         unsigned* status, bool abortable = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  const uint64_t lim = (uint64_t)limit_us * 1000ull;
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255) == 0) {
      if (abortable && *abort_flag) return false;
      if (globaltimer_ns() - t0 > lim) break;
    }
  }
  *abort_flag = 1;
  atomicOr(status, kStatusTimeout);
  return false;
}

struct TileInfo {
  int e, lm, nt, row0, valid;
};

__device__ __forceinline__ TileInfo decode_tile(const Bars& b, int E, int NT, int t) {
  TileInfo ti;
  const int mt = t / NT;
  ti.nt = t - mt * NT;
  int lo = 0, hi = E - 1;  // largest e with mt_off[e] <= mt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (b.mt_off[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  ti.e = lo;
  ti.lm = mt - b.mt_off[lo];
  ti.row0 = b.offsets[lo] + ti.lm * kBM;
  ti.valid = min(kBM, b.counts[lo] - ti.lm * kBM);
  return ti;
}

__device__ __forceinline__ float silu_clamped(float hg, float hu) {
  const float g = fminf(hg, 7.f);
  const float u = fminf(fmaxf(hu, -7.f), 7.f);
  return (u + 1.f) * g * (1.f / (1.f + expf(-1.702f * g)));
}

template <int BN, int STAGES, bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_mxfp4_gemm(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapP,
                       GemmArgs a) {
  using L = Smem<BN, STAGES>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int KB = a.K / 32;
  const int KT = a.K / kBK;
  const int NT = a.N / BN;
  const int scbytes = BN * KB;
  Bars& b = *reinterpret_cast<Bars*>(smem + L::offSC + 2 * scbytes);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* abort_flag = &b.abort_flag;

  for (int i = tid; i < a.E; i += kThreads) b.counts[i] = a.counts[i];
  for (int i = tid; i <= a.E; i += kThreads) {
    b.offsets[i] = a.offsets[i];
    b.mt_off[i] = a.mt_off[i];
  }
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&b.full_ab[s], 1);
      mbar_init(&b.full_b[s], 4);
      mbar_init(&b.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b.sc_full[i], 1);
      mbar_init(&b.sc_empty[i], 4);
      mbar_init(&b.acc_full[i], 1);
      mbar_init(&b.acc_empty[i], 4);
    }
    mbar_init(&b.drain, 1);
    b.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&b.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = b.tmem_base;
  const int total_tiles = b.mt_off[a.E] * NT;
  const long long lim = a.spin_limit;

  if (warp == kProdWarp) {
    if (lane == 0) {
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tc) {
        const TileInfo ti = decode_tile(b, a.E, NT, t);
        const int sb = tc & 1;
        if (tc >= 2) ok = wait_bar(&b.sc_empty[sb], ((tc >> 1) - 1) & 1, lim, abort_flag, a.status);
        if (!ok) break;
        uint8_t* scdst = smem + L::offSC + sb * scbytes;
        mbar_arrive_expect_tx(&b.sc_full[sb], scbytes);
        bulk_load(scdst, a.scales + ((size_t)ti.e * a.N + (size_t)ti.nt * BN) * KB, scbytes, &b.sc_full[sb]);
        const int prow = ti.e * a.N + ti.nt * BN;
        for (int kt = 0; kt < KT; ++kt, ++it) {
          const int s = it % STAGES;
          ok = wait_bar(&b.empty[s], ((it / STAGES) & 1) ^ 1, lim, abort_flag, a.status);
          if (!ok) break;
          mbar_arrive_expect_tx(&b.full_ab[s], L::kA + L::kP);
          tma_load_2d(smem + L::offA + s * L::kA, &mapA, &b.full_ab[s], kt * kBK, ti.row0);
          tma_load_2d(smem + L::offP + s * L::kP, &mapP, &b.full_ab[s], kt * (kBK / 2), prow);
        }
      }
      // Drain: wait (bounded) for copies still in flight before the CTA may exit.
      for (int j = (it > STAGES ? it - STAGES : 0); j < it; ++j)
        wait_bar(&b.full_ab[j % STAGES], (j / STAGES) & 1, lim, abort_flag, a.status, false);
      for (int j = (tc > 2 ? tc - 2 : 0); j < tc; ++j)
        wait_bar(&b.sc_full[j & 1], (j >> 1) & 1, lim, abort_flag, a.status, false);
    }
  } else if (warp >= kDeqWarp0) {
    const int dt = tid - kDeqWarp0 * 32;  // 0..127
    int it = 0, tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tc) {
      const int sb = tc & 1;
      ok = wait_bar(&b.sc_full[sb], (tc >> 1) & 1, lim, abort_flag, a.status);
      if (!ok) break;
      const uint8_t* sc = smem + L::offSC + sb * scbytes;
      for (int kt = 0; kt < KT; ++kt, ++it) {
        const int s = it % STAGES;
        ok = wait_bar(&b.full_ab[s], (it / STAGES) & 1, lim, abort_flag, a.status);
        if (!ok) break;
        const uint8_t* P = smem + L::offP + s * L::kP;
        uint8_t* B = smem + L::offB + s * L::kB;
#pragma unroll 4
        for (int c = dt; c < BN * 8; c += 128) {
          const int r = c >> 3, q = c & 7;
          const uint32_t w = *reinterpret_cast<const uint32_t*>(P + r * 32 + q * 4);
          const uint32_t sv = sc[r * KB + kt * 2 + (q >> 2)];
          *reinterpret_cast<uint4*>(B + r * 128 + ((q ^ (r & 7)) << 4)) = mx_dequant8_bf16(w, sv);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&b.full_b[s]);
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&b.sc_empty[sb]);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(kBM, BN);
      int it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tc) {
        const int ab = tc & 1;
        ok = wait_bar(&b.acc_empty[ab], ((tc >> 1) & 1) ^ 1, lim, abort_flag, a.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + ab * 256;
        for (int kt = 0; kt < KT; ++kt, ++it) {
          const int s = it % STAGES;
          const uint32_t par = (it / STAGES) & 1;
          ok = wait_bar(&b.full_ab[s], par, lim, abort_flag, a.status) &&
               wait_bar(&b.full_b[s], par, lim, abort_flag, a.status);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + L::offA + s * L::kA);
          const uint32_t sbb = smem_u32(smem + L::offB + s * L::kB);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16(d_tmem, smem_desc_k128(sa + kk * 32), smem_desc_k128(sbb + kk * 32), idesc,
                      (kt | kk) ? 1u : 0u);
          umma_commit(&b.empty[s]);
        }
        if (!ok) break;
        umma_commit(&b.acc_full[ab]);
      }
      // Drain the tensor core before TMEM is released.
      umma_commit(&b.drain);
      wait_bar(&b.drain, 0, lim, abort_flag, a.status, false);
    }
  } else {
    // epilogue warps 0..3: warp w owns TMEM lanes / tile rows 32w..32w+31
    const int row_in_tile = warp * 32 + lane;
    int tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++tc) {
      const TileInfo ti = decode_tile(b, a.E, NT, t);
      const int ab = tc & 1;
      ok = wait_bar(&b.acc_full[ab], (tc >> 1) & 1, lim, abort_flag, a.status);
      if (!ok) break;
      tc_fence_after();
      const bool valid = row_in_tile < ti.valid;
      const int prow = ti.row0 + row_in_tile;
      const uint16_t* bias = a.bias + (size_t)ti.e * a.N + (size_t)ti.nt * BN;
      const uint32_t tbase = tmem_base + ((uint32_t)(warp * 32) << 16) + ab * 256;
      int pair = 0;
      float wr = 0.f;
      if (!kGateUp && valid) {
        pair = a.perm[prow];
        wr = a.wroute[pair];
      }
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        tmem_ld16(tbase + c0, r);
        tmem_wait_ld();
        if (valid) {
          const uint4 bv0 = *reinterpret_cast<const uint4*>(bias + c0);
          const uint4 bv1 = *reinterpret_cast<const uint4*>(bias + c0 + 8);
          const uint32_t bw[8] = {bv0.x, bv0.y, bv0.z, bv0.w, bv1.x, bv1.y, bv1.z, bv1.w};
          if (kGateUp) {
            uint32_t o[4];
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              const float a0 = silu_clamped(__uint_as_float(r[4 * p + 0]) + bf16_bits_to_float(bw[2 * p] & 0xFFFF),
                                            __uint_as_float(r[4 * p + 1]) + bf16_bits_to_float(bw[2 * p] >> 16));
              const float a1 =
                  silu_clamped(__uint_as_float(r[4 * p + 2]) + bf16_bits_to_float(bw[2 * p + 1] & 0xFFFF),
                               __uint_as_float(r[4 * p + 3]) + bf16_bits_to_float(bw[2 * p + 1] >> 16));
              o[p] = pack_bf16x2(a0, a1);
            }
            const int I = a.N / 2;
            *reinterpret_cast<uint4*>(a.act_out + (size_t)prow * I + (ti.nt * BN + c0) / 2) =
                make_uint4(o[0], o[1], o[2], o[3]);
          } else {
            float4 y[4];
            float* yf = reinterpret_cast<float*>(y);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint32_t bb = (j & 1) ? (bw[j >> 1] >> 16) : (bw[j >> 1] & 0xFFFF);
              yf[j] = (__uint_as_float(r[j]) + bf16_bits_to_float(bb)) * wr;
            }
            float4* dst = reinterpret_cast<float4*>(a.slot_out + (size_t)pair * a.N + ti.nt * BN + c0);
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = y[j];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&b.acc_empty[ab]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, int esize, const void* ptr, uint64_t inner, uint64_t outer,
                 uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * (uint64_t)esize};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN, int STAGES, bool kGateUp>
cudaError_t launch(const GemmArgs& a, const void* a_ptr, int sm_count, cudaStream_t st) {
  CUtensorMap mapA, mapP;
  if (!make_map_2d(&mapA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a_ptr, a.K, a.total_rows, kBK, kBM,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_map_2d(&mapP, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.blocks, a.K / 2, (uint64_t)a.E * a.N, kBK / 2, BN,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return cudaErrorInvalidValue;
  const size_t smem = smem_total<BN, STAGES>(a.K);
  auto kern = grouped_mxfp4_gemm<BN, STAGES, kGateUp>;
  static int configured_smem = 0;  // raise the limit only when a larger K needs it
  if ((int)smem > configured_smem) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    configured_smem = (int)smem;
  }
  const long long mt_max = ((long long)a.total_rows + kBM - 1) / kBM + a.E;
  const long long tiles_max = mt_max * (a.N / BN);
  const int grid = (int)(tiles_max < sm_count ? tiles_max : sm_count);
  kern<<<grid, kThreads, smem, st>>>(mapA, mapP, a);
  return cudaGetLastError();
}

}  // namespace

int gemm_pick_bn(int N) {
  if (N % 240 == 0) return 240;
  if (N % 192 == 0) return 192;
  if (N % 128 == 0) return 128;
  return 64;
}

template <bool kGateUp>
cudaError_t launch_dispatch(const GemmArgs& a, const void* a_ptr, int sm_count, cudaStream_t st) {
  if (a.K % kBK || a.N % 64) return cudaErrorInvalidValue;
  switch (gemm_pick_bn(a.N)) {
    case 240: return launch<240, 3, kGateUp>(a, a_ptr, sm_count, st);
    case 192: return launch<192, 4, kGateUp>(a, a_ptr, sm_count, st);
    case 128: return launch<128, 4, kGateUp>(a, a_ptr, sm_count, st);
    default: return launch<64, 4, kGateUp>(a, a_ptr, sm_count, st);
  }
}

cudaError_t launch_gemm_gateup(const GemmArgs& a, const void* a_ptr, int sm_count, cudaStream_t st) {
  return launch_dispatch<true>(a, a_ptr, sm_count, st);
}

cudaError_t launch_gemm_down(const GemmArgs& a, const void* a_ptr, int sm_count, cudaStream_t st) {
  return launch_dispatch<false>(a, a_ptr, sm_count, st);
}

}  // namespace moe
