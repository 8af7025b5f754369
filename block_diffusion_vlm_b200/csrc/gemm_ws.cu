// Decoder-layer GEMMs for batch-1 block decoding: y = x . W^T with W streamed
// from HBM once (tcgen05 UMMA, weights as the 128-row operand, token rows as
// N), and the layer's elementwise work fused into the epilogue:
//   EPI_QKV    y * rmsnorm factor -> RoPE (query and key heads) -> bf16;
//              queries to the q buffer, keys/values straight into the KV
//              cache at slots L.. (values transposed);
//   EPI_RESID  residual add x += y (bf16 stream) and the new rows' sums of
//              squares per 128 features (the next RMSNorm's input);
//   EPI_SWIGLU gate/up tile (64 gate rows over 64 up rows) * rmsnorm factor
//              -> silu(g) * u -> bf16 activation.
// Definitions: decoder layer of the Qwen2.5-style language model the method
// converts [Fast-dVLM technical overview (ocdem.com), section 2.1]; the KV
// cache written here is the exact cache of the block-wise decode
// [same page, section 2.2.1].
#include <cstdio>

#include "kernels.h"
#include "mainloop.cuh"

namespace dvlm {

template <int NT, int STAGES>
struct GemmSmem {
  static constexpr int kA = 0;
  static constexpr int kB = kA + STAGES * kATileBytes;
  static constexpr int kE = kB + STAGES * NT * 128;
  static constexpr int kR = kE + 128 * (NT + 1) * 4;
  static constexpr int kBar = kR + 32 * 4;
  static constexpr int kMisc = kBar + (2 * STAGES + 4) * 8;
  static constexpr int kTotal = kMisc + 64 + 1024;  // + alignment slack
};

template <int NT>
struct StagesFor {
  static constexpr int value = NT <= 16 ? 5 : 4;
};

template <int NT, int STAGES, int EPI>
__global__ void __launch_bounds__(kWsThreads, 2)
    gemm_ws_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapA2,
                   const __grid_constant__ CUtensorMap mapB, const SkSched sc, const int a_row_base,
                   const GemmEpi ea) {
  using S = GemmSmem<NT, STAGES>;
  constexpr int TMC = tmem_cols_for<NT>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem + S::kA;
  uint8_t* sB = smem + S::kB;
  float* sE = reinterpret_cast<float*>(smem + S::kE);
  float* sR = reinterpret_cast<float*>(smem + S::kR);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  int* sflag = reinterpret_cast<int*>(smem + S::kMisc + 4);
  volatile int* sabort = reinterpret_cast<volatile int*>(smem + S::kMisc + 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long u0 = sc.begin(blockIdx.x), u1 = sc.begin(blockIdx.x + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], 4);
    }
    *sabort = 0;
    fence_mbar_init();
    tma_prefetch_map(&mapA);
    if (EPI == EPI_SWIGLU) tma_prefetch_map(&mapA2);
    tma_prefetch_map(&mapB);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, TMC);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_launch_dependents();

  if (warp == 0) {
    if (lane == 0 && u1 > u0)
      ws_producer<NT, STAGES, EPI == EPI_SWIGLU>(&mapA, &mapA2, &mapB, sA, sB, full, empty, sc, u0, u1, a_row_base,
                                                 0, ea.status, sabort);
  } else if (warp == 1) {
    if (lane == 0 && u1 > u0) ws_mma<NT, STAGES>(sA, sB, full, empty, accf, acce, tmem, sc, u0, u1, ea.status, sabort);
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // accumulator row = output feature within the tile
    const int et = threadIdx.x - 64;      // 0..127
    griddep_wait();
    if (EPI != EPI_RESID) {
      if (et < NT) {
        float s = 0.f;
        for (int p = 0; p < ea.n_ssq; ++p) s += ea.ssq_in[p * NT + et];
        sR[et] = 1.0f / sqrtf(s * ea.inv_h + ea.eps);
      }
      named_bar_sync(1, 128);
    }
    int L0 = 0;
    if (EPI == EPI_QKV) L0 = ea.d_len ? *ea.d_len : ea.L_static;
    const int first_tile = sc.first_tile(blockIdx.x);
    int seg = 0;
    for (long long u = u0; u < u1; ++seg) {
      const int T = static_cast<int>(u / sc.kb);
      const long long t_begin = static_cast<long long>(T) * sc.kb, t_end = t_begin + sc.kb;
      const long long seg_end = t_end < u1 ? t_end : u1;
      const int b = seg & 1;
      mbar_wait(&accf[b], (seg >> 1) & 1, ea.status, sabort);
      named_bar_sync(1, 128);  // leave together if any wait gave up
      if (*sabort) break;
      tc_fence_after();
      float v[NT];
      ws_load_acc<NT>(tmem, b, quarter, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
      const bool whole = (u == t_begin) && (seg_end == t_end);
      if (!whole) {
        const int slot = (T == first_tile) ? 0 : 1;
        float* mine = ea.part + (static_cast<size_t>(blockIdx.x) * 2 + slot) * NT * 128;
#pragma unroll
        for (int t = 0; t < NT; ++t) __stcg(&mine[t * 128 + row], v[t]);
        __threadfence();
        named_bar_sync(1, 128);
        const int pf = sc.cta_of(t_begin), pl = sc.cta_of(t_end - 1);
        if (et == 0) {
          const int old = atomicAdd(&ea.cnt[T], 1);
          *sflag = (old == pl - pf) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (!*sflag) {
          u = seg_end;
          continue;
        }
        __threadfence();
#pragma unroll
        for (int t = 0; t < NT; ++t) v[t] = 0.f;
        for (int p = pf; p <= pl; ++p) {
          const int sp = (T == sc.first_tile(p)) ? 0 : 1;
          const float* src = ea.part + (static_cast<size_t>(p) * 2 + sp) * NT * 128;
#pragma unroll
          for (int t = 0; t < NT; ++t) v[t] += __ldcg(&src[t * 128 + row]);
        }
        if (et == 0) ea.cnt[T] = 0;
      }

      if (EPI == EPI_RESID) {
        const int col = T * 128 + row;
        float sq[NT];
#pragma unroll
        for (int t = 0; t < NT; ++t) {
          sq[t] = 0.f;
          if (t < ea.n_rows) {
            bf16* px = ea.resid + static_cast<size_t>(t) * ea.resid_ld + col;
            const float xn = bf16_round_f(__bfloat162float(*px) + v[t]);
            *px = __float2bfloat16_rn(xn);
            sq[t] = xn * xn;
          }
          sE[row * (NT + 1) + t] = sq[t];
        }
        named_bar_sync(1, 128);
        if (et < NT) {
          float s = 0.f;
          for (int r = 0; r < 128; ++r) s += sE[r * (NT + 1) + et];
          ea.ssq_out[T * NT + et] = s;
        }
        named_bar_sync(1, 128);
      } else {
#pragma unroll
        for (int t = 0; t < NT; ++t) sE[row * (NT + 1) + t] = v[t] * sR[t];
        named_bar_sync(1, 128);
        const int j = et & 63;
        const int half = et >> 6;
        const int t0 = half * (NT / 2), t1 = t0 + NT / 2;
        if (EPI == EPI_SWIGLU) {
          for (int t = t0; t < t1 && t < ea.n_rows; ++t) {
            const float g = sE[j * (NT + 1) + t];
            const float up = sE[(j + 64) * (NT + 1) + t];
            const float a = g / (1.0f + expf(-g)) * up;
            ea.out[static_cast<size_t>(t) * ea.out_ld + T * 64 + j] = __float2bfloat16_rn(a);
          }
        } else {  // EPI_QKV, one head (128 rows) per tile
          const int nq = ea.n_q_heads, nkv = ea.n_kv_heads;
          if (T < nq + nkv) {
            const double inv_freq = exp2(-(2.0 * j / 128.0) * ea.log2_rope_base);
            for (int t = t0; t < t1 && t < ea.n_rows; ++t) {
              const float x1 = sE[j * (NT + 1) + t];
              const float x2 = sE[(j + 64) * (NT + 1) + t];
              double sn, cs;
              sincos(static_cast<double>(L0 + t) * inv_freq, &sn, &cs);
              const float c = static_cast<float>(cs), s = static_cast<float>(sn);
              const bf16 y1 = __float2bfloat16_rn(x1 * c - x2 * s);
              const bf16 y2 = __float2bfloat16_rn(x2 * c + x1 * s);
              if (T < nq) {
                bf16* q = ea.out + static_cast<size_t>(t) * ea.out_ld + T * 128;
                q[j] = y1;
                q[j + 64] = y2;
              } else {
                bf16* k = ea.kcache + (static_cast<size_t>(T - nq) * ea.Lmax + (L0 + t)) * 128;
                k[j] = y1;
                k[j + 64] = y2;
              }
            }
          } else {
            const int h = T - nq - nkv;
            for (int t = t0; t < t1 && t < ea.n_rows; ++t) {
              ea.vcache[(static_cast<size_t>(h) * 128 + j) * ea.Lmax + (L0 + t)] =
                  __float2bfloat16_rn(sE[j * (NT + 1) + t]);
              ea.vcache[(static_cast<size_t>(h) * 128 + j + 64) * ea.Lmax + (L0 + t)] =
                  __float2bfloat16_rn(sE[(j + 64) * (NT + 1) + t]);
            }
          }
        }
        named_bar_sync(1, 128);
      }
      u = seg_end;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMC);
  }
}

template <int NT, int EPI>
static cudaError_t launch_one(const CUtensorMap& mapA, const CUtensorMap& mapA2, const CUtensorMap& mapB,
                              const SkSched& sc, int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s) {
  constexpr int ST = StagesFor<NT>::value;
  using S = GemmSmem<NT, ST>;
  auto kern = gemm_ws_kernel<NT, ST, EPI>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sc.P);
  cfg.blockDim = dim3(kWsThreads);
  cfg.dynamicSmemBytes = S::kTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mapA, mapA2, mapB, sc, a_row_base, ea);
}

size_t gemm_ws_part_bytes(int NT, int P) { return static_cast<size_t>(P) * 2 * NT * 128 * sizeof(float); }

cudaError_t launch_gemm_ws(int NT, const CUtensorMap& mapA, const CUtensorMap& mapA2, const CUtensorMap& mapB,
                           int n_tiles, int kb, int P, int a_row_base, const GemmEpi& ea, bool pdl,
                           cudaStream_t s) {
  SkSched sc{n_tiles, kb, P};
#define DVLM_GEMM_CASE(nt)                                                                       \
  if (NT == nt) {                                                                                \
    switch (ea.epi) {                                                                            \
      case EPI_QKV: return launch_one<nt, EPI_QKV>(mapA, mapA2, mapB, sc, a_row_base, ea, pdl, s);       \
      case EPI_RESID: return launch_one<nt, EPI_RESID>(mapA, mapA2, mapB, sc, a_row_base, ea, pdl, s);   \
      case EPI_SWIGLU: return launch_one<nt, EPI_SWIGLU>(mapA, mapA2, mapB, sc, a_row_base, ea, pdl, s); \
    }                                                                                            \
  }
  DVLM_GEMM_CASE(16)
  DVLM_GEMM_CASE(32)
#undef DVLM_GEMM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace dvlm
