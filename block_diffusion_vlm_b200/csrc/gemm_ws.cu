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

// Activation code blocks an fp8 CTA can hold (its k range, 128 wide each).
constexpr int kMaxFp8Blocks = 16;

template <int NT, int STAGES, bool FP8 = false>
struct GemmSmem {
  static constexpr int kA = 0;
  static constexpr int kB = kA + STAGES * kATileBytes;
  static constexpr int kE = kB + (FP8 ? kMaxFp8Blocks : STAGES) * NT * 128;
  static constexpr int kR = kE + 128 * (NT + 1) * 4;
  static constexpr int kAt = kR + 32 * 4;  // fp8: token scales [32], quantisation multipliers [32], amax [32]
  static constexpr int kBar = kAt + 3 * 32 * 4;
  static constexpr int kMisc = kBar + (2 * STAGES + 8) * 8;  // + the persistent forward's attention barriers
  static constexpr int kTotal = kMisc + 64 + 1024;  // + alignment slack
};

// Per-row scale of an E4M3 weight tile row (absolute weight row index).
__device__ __forceinline__ float fp8_row_scale(const GemmEpi& ea, bool split, int a_row_base, int T, int row) {
  if (split) return row < 64 ? ea.wscale[a_row_base + T * 64 + row] : ea.wscale2[a_row_base + T * 64 + row - 64];
  return ea.wscale[a_row_base + T * 128 + row];
}

// RMSNorm factors of the NT input rows from the producers' per-tile sums of
// squares (ssq_in [n_ssq][NT]), run by the 128 epilogue threads: 128 / NT
// partial sums per row, each thread's loads issued together (up to 16 of
// them in flight), then one thread per row adds the partials in order.
// sPart: 128 floats of scratch.
template <int NT>
__device__ __forceinline__ void rms_factors(const float* ssq_in, int n_ssq, float inv_h, float eps, int et,
                                            float* sR, float* sPart) {
  constexpr int G = 128 / NT;
  constexpr int BATCH = 16;
  const int t = et % NT, g = et / NT;
  float s = 0.f;
  for (int q0 = g; q0 < n_ssq; q0 += G * BATCH) {
    float v[BATCH];
#pragma unroll
    for (int j = 0; j < BATCH; ++j) {
      const int q = q0 + j * G;
      v[j] = q < n_ssq ? __ldcg(&ssq_in[q * NT + t]) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < BATCH; ++j) s += v[j];
  }
  sPart[g * NT + t] = s;
  named_bar_sync(1, 128);
  if (et < NT) {
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < G; ++k) tot += sPart[k * NT + et];
    sR[et] = 1.0f / sqrtf(tot * inv_h + eps);
  }
  named_bar_sync(1, 128);
}
template <int NT>
__device__ __forceinline__ void ws_rms_factors(const GemmEpi& ea, int et, float* sR, float* sPart) {
  rms_factors<NT>(ea.ssq_in, ea.n_ssq, ea.inv_h, ea.eps, et, sR, sPart);
}

// The epilogue warps' work for the stream-K units [u0, u1) of one GEMM:
// partial tiles stored for the CTAs that finish them, split tiles finished
// (partials added in CTA order), the fused epilogue on every tile this CTA
// owns.  gseg counts the CTA's segments across consecutive GEMMs (it selects
// the accumulator buffer and its phase); L0 is the QKV rows' first slot.
// Returns false when a wait gave up.
template <int NT, int EPI, bool FP8>
__device__ __forceinline__ bool ws_epilogue_units(const SkSched& sc, long long u0, long long u1, int a_row_base,
                                                  const GemmEpi& ea, uint32_t tmem, uint64_t* accf,
                                                  uint64_t* acce, float* sE, const float* sR, const float* sAt,
                                                  unsigned* sAmax, int* sflag, volatile int* sabort, int& gseg,
                                                  int L0) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;  // accumulator row = output feature within the tile
  const int et = threadIdx.x - 64;      // 0..127
  // A tile split over CTAs pf < ... < pl is finished by pf, which streams
  // the tile's first k blocks as its last segment; the others stream their
  // parts first and leave fp32 partials in global scratch, counted on
  // cnt[T].  pf fetches those partials while its own last segment is still
  // in the mainloop and adds them in CTA order.
  for (long long u = u0; u < u1; ++gseg) {
    const int T = static_cast<int>(u / sc.kb);
    const long long t_begin = static_cast<long long>(T) * sc.kb, t_end = t_begin + sc.kb;
    const long long seg_end = t_end < u1 ? t_end : u1;
    const int b = gseg & 1;
    const bool whole = (u == t_begin) && (seg_end == t_end);
    const bool finisher = !whole && (u == t_begin);
    float o[NT];
    // residual rows of the tile's columns, fetched before the accumulator is
    // ready (independent loads; only this tile's epilogue writes them)
    float xr[NT];
    if (EPI == EPI_RESID && (whole || finisher)) {
      const int col = T * 128 + row;
#pragma unroll
      for (int t = 0; t < NT; ++t)
        xr[t] = t < ea.n_rows ? __bfloat162float(__ldcg(ea.resid + static_cast<size_t>(t) * ea.resid_ld + col)) : 0.f;
    }
    if (finisher) {
      const int pl = sc.cta_of(t_end - 1);
      if (et == 0) {
        const bool ok = wait_counter(&ea.cnt[T], pl - static_cast<int>(blockIdx.x), ea.status, sabort);
        if (ok) ea.cnt[T] = 0;  // every part is counted: zero again for the next launch
        *sflag = ok ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (!*sflag) return false;
      __threadfence();
#pragma unroll
      for (int t = 0; t < NT; ++t) o[t] = 0.f;
      // the other CTAs' partials in CTA order, four sources' loads in flight
      for (int p0 = static_cast<int>(blockIdx.x) + 1; p0 <= pl; p0 += 4) {
        float q4[4][NT];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float* src = ea.part + static_cast<size_t>(p0 + q <= pl ? p0 + q : p0) * NT * 128;
#pragma unroll
          for (int t = 0; t < NT; ++t) q4[q][t] = __ldcg(&src[t * 128 + row]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (p0 + q <= pl) {
#pragma unroll
            for (int t = 0; t < NT; ++t) o[t] += q4[q][t];
          }
      }
    }
    mbar_wait(&accf[b], (gseg >> 1) & 1, ea.status, sabort);
    named_bar_sync(1, 128);  // leave together if any wait gave up
    if (*sabort) return false;
    tc_fence_after();
    float v[NT];
    ws_load_acc<NT>(tmem, b, quarter, v, seg_end - u >= 2);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&acce[b]);
    if (!whole && !finisher) {
      // tail or middle part of a tile finished by another CTA
      float* mine = ea.part + static_cast<size_t>(blockIdx.x) * NT * 128;
#pragma unroll
      for (int t = 0; t < NT; ++t) __stcg(&mine[t * 128 + row], v[t]);
      __threadfence();
      named_bar_sync(1, 128);
      if (et == 0) red_release_gpu_add(&ea.cnt[T], 1);
      u = seg_end;
      continue;
    }
    if (finisher) {
#pragma unroll
      for (int t = 0; t < NT; ++t) v[t] += o[t];
    }
    if (FP8) {  // W8A8 dequantisation: weight row scale x token scale
      const float sr = fp8_row_scale(ea, EPI == EPI_SWIGLU, a_row_base, T, row);
#pragma unroll
      for (int t = 0; t < NT; ++t) v[t] *= sr * sAt[t];
    }

    if (EPI == EPI_RESID) {
      const int col = T * 128 + row;
      float sq[NT];
#pragma unroll
      for (int t = 0; t < NT; ++t) {
        sq[t] = 0.f;
        if (t < ea.n_rows) {
          const float xn = bf16_round_f(xr[t] + v[t]);
          ea.resid[static_cast<size_t>(t) * ea.resid_ld + col] = __float2bfloat16_rn(xn);
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
      for (int t = 0; t < NT; ++t) sE[row * (NT + 1) + t] = FP8 ? v[t] : v[t] * sR[t];
      if (FP8 && EPI == EPI_SWIGLU && et < NT) sAmax[et] = 0u;
      named_bar_sync(1, 128);
      const int j = et & 63;
      const int half = et >> 6;
      const int t0 = half * (NT / 2), t1 = t0 + NT / 2;
      if (EPI == EPI_SWIGLU) {
        for (int t = t0; t < t1 && t < ea.n_rows; ++t) {
          const float g = sE[j * (NT + 1) + t];
          const float up = sE[(j + 64) * (NT + 1) + t];
          const float a = g / (1.0f + expf(-g)) * up;
          const bf16 ab = __float2bfloat16_rn(a);
          ea.out[static_cast<size_t>(t) * ea.out_ld + T * 64 + j] = ab;
          if (FP8) atomicMax(&sAmax[t], __float_as_uint(fabsf(__bfloat162float(ab))));
        }
        if (FP8) {
          named_bar_sync(1, 128);
          if (et < NT) ea.amax_out[T * NT + et] = __uint_as_float(sAmax[et]);
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
            } else if (bf16* k = kv_k_ptr(ea, T - nq, L0 + t)) {
              k[j] = y1;
              k[j + 64] = y2;
            } else {
              record_error(ea.status, DVLM_ERR_BOUNDS);
            }
          }
        } else {
          const int h = T - nq - nkv;
          for (int t = t0; t < t1 && t < ea.n_rows; ++t) {
            bf16* v1 = kv_v_ptr(ea, h, j, L0 + t);
            bf16* v2 = kv_v_ptr(ea, h, j + 64, L0 + t);
            if (!v1 || !v2) {
              record_error(ea.status, DVLM_ERR_BOUNDS);
              continue;
            }
            *v1 = __float2bfloat16_rn(sE[j * (NT + 1) + t]);
            *v2 = __float2bfloat16_rn(sE[(j + 64) * (NT + 1) + t]);
          }
        }
      }
      named_bar_sync(1, 128);
    }
    u = seg_end;
  }
  return true;
}

template <int NT, int STAGES, int EPI, bool FP8 = false>
__global__ void __launch_bounds__(kWsThreads, NT <= 16 ? 2 : 1)
    gemm_ws_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapA2,
                   const __grid_constant__ CUtensorMap mapB, const SkSched sc, const int a_row_base,
                   const GemmEpi ea) {
  using S = GemmSmem<NT, STAGES, FP8>;
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
  uint64_t* b_ready = acce + 2;  // fp8: the activation codes are in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  int* sflag = reinterpret_cast<int*>(smem + S::kMisc + 4);
  volatile int* sabort = reinterpret_cast<volatile int*>(smem + S::kMisc + 8);
  float* sAt = reinterpret_cast<float*>(smem + S::kAt);
  float* sQm = sAt + 32;
  unsigned* sAmax = reinterpret_cast<unsigned*>(sAt + 64);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long u0 = sc.begin(blockIdx.x), u1 = sc.begin(blockIdx.x + 1);
  // fp8: 128-wide k blocks whose activation codes this CTA needs
  int kb_lo = 0, kb_hi = sc.kb;
  if (FP8 && u1 > u0 && u0 / sc.kb == (u1 - 1) / sc.kb) {
    kb_lo = static_cast<int>(u0 % sc.kb);
    kb_hi = static_cast<int>((u1 - 1) % sc.kb) + 1;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 2);
      mbar_init(&acce[b], 4);
    }
    mbar_init(b_ready, 1);
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

  if (warp == 0) {
    if (lane == 0 && u1 > u0)
      ws_producer<NT, STAGES, EPI == EPI_SWIGLU, FP8>(&mapA, &mapA2, &mapB, sA, sB, full, empty, sc, u0, u1,
                                                      a_row_base, 0, ea.status, sabort);
  } else if (warp == 1 || warp == kMmaWarp2) {
    if (lane == 0 && u1 > u0)
      ws_mma<NT, STAGES, FP8>(sA, sB, full, empty, accf, acce, tmem, sc, u0, u1, ea.status, sabort,
                              warp == 1 ? 0 : 1, b_ready, kb_lo);
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // accumulator row = output feature within the tile
    const int et = threadIdx.x - 64;      // 0..127
    griddep_wait();
    // Dependents may start only once this kernel's own inputs are complete,
    // so at most two kernels of the chain overlap (see ptx.cuh).
    if (et == 0) griddep_launch_dependents();
    if (EPI != EPI_RESID) ws_rms_factors<NT>(ea, et, sR, sE);
    if (FP8)
      fp8_quantize_activations<NT>(et, ea.q_src, ea.q_ld, ea.q_K, ea.n_rows, ea.rms_input ? sR : nullptr,
                                   ea.amax_in, ea.n_amax, kb_lo, kb_hi, sB, sAt, sQm, b_ready);
    int L0 = 0;
    if (EPI == EPI_QKV) L0 = ea.d_len ? *ea.d_len : ea.L_static;
    int gseg = 0;
    ws_epilogue_units<NT, EPI, FP8>(sc, u0, u1, a_row_base, ea, tmem, accf, acce, sE, sR, sAt, sAmax, sflag,
                                    sabort, gseg, L0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMC);
  }
}

// ---------------------------------------------------------------------------
// Cluster split-K variant for the narrow projections (QKV, O-proj, down):
// one output tile per cluster of S CTAs, CTA c streaming the contiguous k
// range [c*kb/S, (c+1)*kb/S).  The S fp32 partial tiles meet in distributed
// shared memory and every CTA finishes a slice of the tile's rows, summing
// the partials in rank order (deterministic; each token column's arithmetic
// is independent of how many rows the step has).
template <int NT, int STAGES, bool FP8 = false>
struct ClSmem {
  static constexpr int kA = 0;
  static constexpr int kB = kA + STAGES * kATileBytes;
  static constexpr int kSend = kB + (FP8 ? kMaxFp8Blocks : STAGES) * NT * 128;  // partial tile [128][NT] fp32
  static constexpr int kRecv = kSend + 128 * NT * 4;    // slices received [S][rows][NT] (<= 160 rows)
  static constexpr int kQ = kRecv + 160 * NT * 4;       // squares of this CTA's rows [64][NT+1]
  static constexpr int kR = kQ + 64 * (NT + 1) * 4;     // rmsnorm factors [NT]
  static constexpr int kAt = kR + 32 * 4;               // fp8: token scales [32], multipliers [32]
  static constexpr int kBar = kAt + 2 * 32 * 4;
  static constexpr int kMisc = kBar + (2 * STAGES + 6) * 8;
  static constexpr int kTotal = kMisc + 64 + 1024;
};

template <int NT, int STAGES, int EPI, bool FP8 = false>
__global__ void __launch_bounds__(kWsThreads, NT <= 16 ? 2 : 1)
    gemm_cl_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB, const int kb,
                   const int S, const int a_row_base, const GemmEpi ea) {
  using Sm = ClSmem<NT, STAGES, FP8>;
  constexpr int TMC = tmem_cols_for<NT>();
  constexpr int PS = NT + 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem + Sm::kA;
  uint8_t* sB = smem + Sm::kB;
  float* sSend = reinterpret_cast<float*>(smem + Sm::kSend);
  float* sRecv = reinterpret_cast<float*>(smem + Sm::kRecv);
  float* sQ = reinterpret_cast<float*>(smem + Sm::kQ);
  float* sR = reinterpret_cast<float*>(smem + Sm::kR);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Sm::kBar);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint64_t* recv_full = acce + 2;  // every cluster CTA's slice of this CTA's rows landed
  uint64_t* b_ready = recv_full + 1;  // fp8: the activation codes are in shared memory
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Sm::kMisc);
  volatile int* sabort = reinterpret_cast<volatile int*>(smem + Sm::kMisc + 8);
  float* sAt = reinterpret_cast<float*>(smem + Sm::kAt);
  float* sQm = sAt + 32;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c = static_cast<int>(cluster_ctarank());
  const int T = blockIdx.x / S;
  const SkSched sc{static_cast<int>(gridDim.x) / S, kb, 1};
  const long long u0 = static_cast<long long>(T) * kb + static_cast<long long>(c) * kb / S;
  const long long u1 = static_cast<long long>(T) * kb + static_cast<long long>(c + 1) * kb / S;
  // Rows of the tile finished by cluster CTA d: RESID rows [a0, a0+n); QKV the
  // RoPE pairs (j, j+64) for j in [a0, a0+n), so a pair never straddles CTAs.
  auto slice = [&](int d, int& a0, int& n) {
    const int span = EPI == EPI_RESID ? 128 : 64;
    a0 = d * span / S;
    n = (d + 1) * span / S - a0;
  };
  constexpr int kPieces = EPI == EPI_RESID ? 1 : 2;  // row ranges per slice
  int my0, myn;
  slice(c, my0, myn);
  // slice elements per epilogue thread: at most 64 rows (S >= 2) x NT over 128
  constexpr int kMaxPer = (64 * NT + 127) / 128;
  // The cache length is final before this kernel's predecessor runs.
  const int L0 = (EPI == EPI_QKV) ? (ea.d_len ? *ea.d_len : ea.L_static) : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 2);
      mbar_init(&acce[b], 4);
    }
    mbar_init(recv_full, 1);
    mbar_init(b_ready, 1);
    *sabort = 0;
    fence_mbar_init();
    mbar_arrive_expect_tx(recv_full, static_cast<uint32_t>(S * kPieces * myn * NT * 4));
    tma_prefetch_map(&mapA);
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
  // Receive barriers initialised cluster-wide before any CTA sends (waited on
  // just before the sends).
  cluster_arrive();

  const int et = threadIdx.x - 64;  // epilogue thread 0..127 (warps 2..5)
  float pre_a[kMaxPer], pre_b[kMaxPer];
  const int kb_lo = c * kb / S, kb_hi = (c + 1) * kb / S;  // fp8: this CTA's k blocks
  if (warp == 0) {
    if (lane == 0 && u1 > u0)
      ws_producer<NT, STAGES, false, FP8>(&mapA, &mapA, &mapB, sA, sB, full, empty, sc, u0, u1, a_row_base, 0,
                                          ea.status, sabort);
  } else if (warp == 1 || warp == kMmaWarp2) {
    if (lane == 0 && u1 > u0)
      ws_mma<NT, STAGES, FP8>(sA, sB, full, empty, accf, acce, tmem, sc, u0, u1, ea.status, sabort,
                              warp == 1 ? 0 : 1, b_ready, kb_lo);
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    griddep_wait();
    // Dependents may start only once this kernel's own inputs are complete,
    // so at most two kernels of the chain overlap (see ptx.cuh).
    if (et == 0) griddep_launch_dependents();
    if (EPI == EPI_QKV) rms_factors<NT>(ea.ssq_in, ea.n_ssq, ea.inv_h, ea.eps, et, sR, sQ);
    if (FP8)
      fp8_quantize_activations<NT>(et, ea.q_src, ea.q_ld, ea.q_K, ea.n_rows, ea.rms_input ? sR : nullptr,
                                   ea.amax_in, ea.n_amax, kb_lo, kb_hi, sB, sAt, sQm, b_ready);
    // Operands of this thread's share of the slice epilogue that do not
    // depend on the product, fetched while the mainloop streams: the residual
    // entries (RESID) or the RoPE rotation (QKV).
#pragma unroll
    for (int k = 0; k < kMaxPer; ++k) {
      const int it = et + 128 * k;
      pre_a[k] = 0.f;
      pre_b[k] = 0.f;
      if (it >= myn * NT) continue;
      const int t = it % NT;
      if (t >= ea.n_rows) continue;
      if (EPI == EPI_RESID) {
        pre_a[k] = __bfloat162float(ea.resid[static_cast<size_t>(t) * ea.resid_ld + T * 128 + my0 + it / NT]);
      } else if (T < ea.n_q_heads + ea.n_kv_heads) {
        const int j = my0 + it / NT;
        const double inv_freq = exp2(-(2.0 * j / 128.0) * ea.log2_rope_base);
        double sn, cs;
        sincos(static_cast<double>(L0 + t) * inv_freq, &sn, &cs);
        pre_a[k] = static_cast<float>(cs);
        pre_b[k] = static_cast<float>(sn);
      }
    }
    float v[NT];
    if (u1 > u0) {
      mbar_wait(&accf[0], 0, ea.status, sabort);
      tc_fence_after();
      ws_load_acc<NT>(tmem, 0, quarter, v, u1 - u0 >= 2);
    } else {
#pragma unroll
      for (int t = 0; t < NT; ++t) v[t] = 0.f;
    }
    float4* s4 = reinterpret_cast<float4*>(sSend + row * NT);
#pragma unroll
    for (int t = 0; t < NT; t += 4) s4[t / 4] = make_float4(v[t], v[t + 1], v[t + 2], v[t + 3]);
    // Slice d of the partial goes to cluster CTA d, which sums the S partials
    // of its rows: bulk copies into that CTA's receive buffer (source-major),
    // counted on its receive barrier.
    fence_proxy_async_smem();
    named_bar_sync(1, 128);
    cluster_wait();
    if (et < S) {
      int a0, n;
      slice(et, a0, n);
      if (n > 0) {
        const uint32_t rb = map_to_cta(smem_u32(recv_full), et);
        const uint32_t bytes = static_cast<uint32_t>(n * NT * 4);
        const uint32_t dst = map_to_cta(smem_u32(sRecv), et) + static_cast<uint32_t>(c * kPieces) * bytes;
        bulk_s2s_cluster(dst, sSend + a0 * NT, bytes, rb);
        if (EPI == EPI_QKV) bulk_s2s_cluster(dst + bytes, sSend + (a0 + 64) * NT, bytes, rb);
      }
      bulk_commit();
    }
  }
  if (warp < 2 || warp == kMmaWarp2) {
    __syncwarp();
    cluster_wait();
  }
  // Every CTA has issued its copies once all have arrived here: a CTA leaves
  // only after that (second barrier, waited on at exit).
  cluster_arrive();

  if (warp >= 2 && warp < kMmaWarp2) {
    const bool got = mbar_wait(recv_full, 0, ea.status, sabort);
    const int rps = kPieces * myn;  // rows from each source
    // Sum of the S partials of element (rl, t) of this CTA's slice, in rank order.
    auto part_sum = [&](int rl, int t) {
      float acc = 0.f;
      for (int q = 0; q < S; ++q) acc += sRecv[(q * rps + rl) * NT + t];
      return acc;
    };
    if (EPI == EPI_RESID) {
#pragma unroll
      for (int k = 0; k < kMaxPer; ++k) {
        const int it = et + 128 * k;
        if (it >= myn * NT) break;
        const int rl = it / NT, t = it % NT;
        float y = got ? part_sum(rl, t) : 0.f;
        if (FP8) y *= ea.wscale[a_row_base + T * 128 + my0 + rl] * sAt[t];
        float sq = 0.f;
        if (t < ea.n_rows) {
          const float xn = bf16_round_f(pre_a[k] + y);
          ea.resid[static_cast<size_t>(t) * ea.resid_ld + T * 128 + my0 + rl] = __float2bfloat16_rn(xn);
          sq = xn * xn;
        }
        sQ[rl * PS + t] = sq;
      }
      named_bar_sync(1, 128);
      // Sums of squares per (tile, cluster CTA): the next RMSNorm adds all
      // n_tiles * S of them in order.
      if (et < NT) {
        float s2 = 0.f;
        for (int rl = 0; rl < myn; ++rl) s2 += sQ[rl * PS + et];
        ea.ssq_out[(T * S + c) * NT + et] = s2;
      }
    } else {  // EPI_QKV: pairs (j, j+64) of one head per tile
      const int nq = ea.n_q_heads, nkv = ea.n_kv_heads;
#pragma unroll
      for (int k = 0; k < kMaxPer; ++k) {
        const int it = et + 128 * k;
        if (it >= myn * NT) break;
        const int jl = it / NT, t = it % NT;
        const int j = my0 + jl;
        const float f1 = FP8 ? ea.wscale[a_row_base + T * 128 + j] * sAt[t] : sR[t];
        const float f2 = FP8 ? ea.wscale[a_row_base + T * 128 + j + 64] * sAt[t] : sR[t];
        const float x1 = (got ? part_sum(jl, t) : 0.f) * f1;
        const float x2 = (got ? part_sum(myn + jl, t) : 0.f) * f2;
        if (t >= ea.n_rows) continue;
        if (T < nq + nkv) {
          const float co = pre_a[k], si = pre_b[k];
          const bf16 y1 = __float2bfloat16_rn(x1 * co - x2 * si);
          const bf16 y2 = __float2bfloat16_rn(x2 * co + x1 * si);
          bf16* dst = (T < nq) ? ea.out + static_cast<size_t>(t) * ea.out_ld + T * 128 : kv_k_ptr(ea, T - nq, L0 + t);
          if (!dst) {
            record_error(ea.status, DVLM_ERR_BOUNDS);
            continue;
          }
          dst[j] = y1;
          dst[j + 64] = y2;
        } else {
          const int h = T - nq - nkv;
          bf16* v1 = kv_v_ptr(ea, h, j, L0 + t);
          bf16* v2 = kv_v_ptr(ea, h, j + 64, L0 + t);
          if (!v1 || !v2) {
            record_error(ea.status, DVLM_ERR_BOUNDS);
            continue;
          }
          *v1 = __float2bfloat16_rn(x1);
          *v2 = __float2bfloat16_rn(x2);
        }
      }
    }
    if (et < S) bulk_wait_read_all();
  }
  tc_fence_before();
  cluster_wait();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMC);
  }
}

// ---------------------------------------------------------------------------
// Persistent forward.  All decoder layers of one forward run in a single
// launch on every SM, phase by phase: the first layer's QKV, then for each
// layer l the attention partials, the attention merge, the O-projection
// (+ residual), gate/up (SwiGLU), down (+ residual) and layer l+1's QKV.  A
// phase reads what the previous phase's epilogues wrote (all CTAs), so a
// grid barrier separates the phases: every CTA bumps a counter after its
// phase epilogue, and phase p's inputs are ready once the counter reaches
// p * gridDim.x.
//
// The weight stream never waits for a barrier: the A loader runs through the
// phases back to back, so while one phase's split tiles are being reduced,
// or the merge runs, or attention computes, the next phases' weight tiles
// are already filling the pipeline stages.  Loads that depend on a phase's
// inputs (a GEMM's activation tiles; attention's query, key and value
// tiles) come from a loader warp of their own that waits for the barrier.
// One A-loader arrival per stage arms the stage's full barrier with all of
// the stage's bytes (a copy from the other loader may complete before that
// arrival; the phase still needs the arrival).
//
// Attention [Fast-dVLM technical overview (ocdem.com), section 2.2.1:
// N2N / N2C / C2C visibility]: units of (KV head g, 64-key chunk c), dealt
// round robin over the CTAs.  A unit takes five pipeline stages -- the
// query tile (8 heads x 16 rows = 128 rows, two 64-wide halves), the
// chunk's keys, its values (transposed) and P -- and leaves, for each row,
// the chunk's unnormalised output O_c = sum_k p_k v_k with p_k = 2^(s_k - m_c)
// (P and V in fp16 for the second product; l_c sums the same fp16 values),
// the row max m_c and l_c.  The
// merge phase combines a row's chunks in chunk order:
// out = sum_c 2^(m_c - M) O_c / sum_c 2^(m_c - M) l_c.  A row's arithmetic
// depends only on its own query and keys (chunks by absolute key position),
// so a 1-row pass and a 16-row pass give bitwise the same rows.
//
// Roles (256 threads): warp 0 A loader, warps 1 and 6 MMA issuers (warp 1
// issues attention too), warps 2..5 epilogue / softmax / merge, warp 7 B
// loader.  All CTAs must be resident at once (one per SM; the launcher checks
// the occupancy), and every wait is bounded: a CTA that gives up records
// DVLM_ERR_TIMEOUT and still arrives at the remaining barriers.
constexpr int kFwdThreads = 256;
constexpr int kFwdStages = 12;
constexpr int kFwdNT = 16;
constexpr int kAttKeys = 64;   // keys per attention unit
constexpr int kAttSlots = 5;   // stages of an attention unit: Q (2 halves), K, V^T, P
constexpr uint32_t kAttIdescS = idesc_bf16_f32(128, kAttKeys);
constexpr uint32_t kAttIdescO = idesc_f16_f32(128, 128);  // P and V in fp16
constexpr int kFwdTmem = 256;  // GEMM accumulators [0, 64), S [64, 128), O [128, 256)
constexpr uint32_t kTmemS = 64, kTmemO = 128;

enum FwdKind { FK_QKV = 0, FK_ATT, FK_MERGE, FK_O, FK_GU, FK_DOWN };

// Kind and layer of phase p.
__device__ __forceinline__ int fwd_kind(const FwdProgram& fp, int p, int& layer) {
  if (p == 0) {
    layer = fp.layer0;
    return FK_QKV;
  }
  const int q = p - 1, r = q % 6;
  layer = fp.layer0 + q / 6 + (r == 5 ? 1 : 0);
  return r == 0 ? FK_ATT : r == 1 ? FK_MERGE : r == 2 ? FK_O : r == 3 ? FK_GU : r == 4 ? FK_DOWN : FK_QKV;
}
__device__ __forceinline__ const ChainPhase& fwd_gemm(const FwdProgram& fp, int kind) {
  return kind == FK_QKV ? fp.qkv : kind == FK_O ? fp.o : kind == FK_GU ? fp.gu : fp.down;
}
__device__ __forceinline__ int fwd_row_base(const FwdProgram& fp, int kind, int layer) {
  return layer * (kind == FK_QKV ? fp.qkv_rows : kind == FK_GU ? fp.I : fp.H);
}
// Cache length of the forward (the previous kernels have completed).
__device__ __forceinline__ int fwd_cache_len(const FwdProgram& fp) {
  griddep_wait();
  return fp.qkv.ea.d_len ? *fp.qkv.ea.d_len : fp.qkv.ea.L_static;
}
__device__ __forceinline__ int att_chunks(const FwdProgram& fp, int L) {
  return (L + fp.qkv.ea.n_rows + kAttKeys - 1) / kAttKeys;
}

// A phase's stream-K schedule: its units over min(P, units) CTAs (a CTA with
// an empty range between the CTAs of a split tile would be counted as one of
// its contributors); CTAs past those have no units in the phase.
__device__ __forceinline__ SkSched chain_sched(const ChainPhase& ph, int P) {
  const long long units = static_cast<long long>(ph.n_tiles) * ph.kb;
  const int ctas = ph.ctas > 0 && ph.ctas < P ? ph.ctas : P;
  return SkSched{ph.n_tiles, ph.kb, static_cast<int>(units < ctas ? units : ctas)};
}
__device__ __forceinline__ void chain_range(const SkSched& sc, long long& u0, long long& u1) {
  if (static_cast<int>(blockIdx.x) >= sc.P) {
    u0 = u1 = 0;
    return;
  }
  u0 = sc.begin(blockIdx.x);
  u1 = sc.begin(blockIdx.x + 1);
}

template <int STAGES>
__device__ __forceinline__ void fwd_load_a(const FwdProgram& fp, uint8_t* sA, uint64_t* full, uint64_t* empty,
                                           volatile int* abort_flag) {
  constexpr int B_BYTES = kFwdNT * 128;
  const uint64_t pol_w = l2_policy_evict_first();
  const int n_phases = 6 * fp.n_layers;
  long long i = 0;
  int L = -1;
  // the next stage, once its previous contents are consumed; arms its full
  // barrier for `bytes` (0: a plain arrival, the stage P of attention)
  auto take = [&](int bytes) -> int {
    const int s = static_cast<int>(i % STAGES);
    if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, fp.status, abort_flag)) return -1;
    if (bytes)
      mbar_arrive_expect_tx(&full[s], bytes);
    else
      mbar_arrive(&full[s]);
    ++i;
    return s;
  };
  for (int p = 0; p < n_phases; ++p) {
    int layer;
    const int kind = fwd_kind(fp, p, layer);
    if (kind == FK_MERGE) continue;
    if (kind == FK_ATT) {
      if (L < 0) L = fwd_cache_len(fp);
      const int n_units = fp.Hkv * att_chunks(fp, L);
      for (int u = blockIdx.x; u < n_units; u += gridDim.x)
        for (int j = 0; j < kAttSlots; ++j)
          if (take(j < kAttSlots - 1 ? kATileBytes : 0) < 0) return;
      continue;
    }
    const ChainPhase& ph = fwd_gemm(fp, kind);
    const int base = fwd_row_base(fp, kind, layer);
    const SkSched sc = chain_sched(ph, gridDim.x);
    long long u0, u1;
    chain_range(sc, u0, u1);
    const bool split = kind == FK_GU;
    for (long long u = u0; u < u1; ++u) {
      const int s = take(kATileBytes + B_BYTES);
      if (s < 0) return;
      const int T = static_cast<int>(u / sc.kb), kk = static_cast<int>(u % sc.kb);
      if (split) {
        tma_load_2d(sA + s * kATileBytes, &ph.mapA, &full[s], kk * 64, base + T * 64, pol_w);
        tma_load_2d(sA + s * kATileBytes + kATileBytes / 2, &ph.mapA2, &full[s], kk * 64, base + T * 64, pol_w);
      } else {
        tma_load_2d(sA + s * kATileBytes, &ph.mapA, &full[s], kk * 64, base + T * 128, pol_w);
      }
    }
  }
}

template <int STAGES>
__device__ __forceinline__ void fwd_load_b(const FwdProgram& fp, uint8_t* sA, uint8_t* sB, uint64_t* full,
                                           uint64_t* empty, volatile int* abort_flag) {
  constexpr int B_BYTES = kFwdNT * 128;
  const uint64_t pol_x = l2_policy_evict_last();
  const int n_phases = 6 * fp.n_layers;
  long long i = 0;
  int L = -1;
  auto next = [&]() -> int {  // the next stage, once its previous contents are consumed
    const int s = static_cast<int>(i % STAGES);
    if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, fp.status, abort_flag)) return -1;
    ++i;
    return s;
  };
  for (int p = 0; p < n_phases; ++p) {
    int layer;
    const int kind = fwd_kind(fp, p, layer);
    // inputs of phase p: the kernel before this one (p = 0), else every CTA's phase p-1
    if (p == 0)
      griddep_wait();
    else if (!wait_counter(fp.bar, p * static_cast<int>(gridDim.x), fp.status, abort_flag))
      return;
    fence_proxy_async_global();
    if (kind == FK_MERGE) continue;
    if (kind == FK_ATT) {
      if (L < 0) L = fwd_cache_len(fp);
      const int n_chunks = att_chunks(fp, L);
      const int n_units = fp.Hkv * n_chunks;
      for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int g = u / n_chunks, c = u % n_chunks;
        const int entry = layer * fp.Hkv + g;  // (layer, KV head) of the cache
        for (int j = 0; j < 2; ++j) {          // query halves: 16 rows x 8 heads x 64
          const int s = next();
          if (s < 0) return;
          tma_load_3d(sA + s * kATileBytes, &fp.mapQ, &full[s], j * 64, g * 8, 0, pol_x);
        }
        int s = next();  // keys of the chunk, two 64-wide halves
        if (s < 0) return;
        const int krow = entry * fp.Lmax + c * kAttKeys;
        tma_load_2d(sA + s * kATileBytes, &fp.mapK, &full[s], 0, krow, pol_x);
        tma_load_2d(sA + s * kATileBytes + kATileBytes / 2, &fp.mapK, &full[s], 64, krow, pol_x);
        s = next();  // values, transposed: 128 rows (d) x 64 keys
        if (s < 0) return;
        tma_load_2d(sA + s * kATileBytes, &fp.mapV, &full[s], c * kAttKeys, entry * 128, pol_x);
        if (next() < 0) return;  // P: written by the softmax warps
      }
      continue;
    }
    const ChainPhase& ph = fwd_gemm(fp, kind);
    const SkSched sc = chain_sched(ph, gridDim.x);
    long long u0, u1;
    chain_range(sc, u0, u1);
    for (long long u = u0; u < u1; ++u) {
      const int s = next();
      if (s < 0) return;
      tma_load_2d(sB + s * B_BYTES, &ph.mapB, &full[s], static_cast<int>(u % sc.kb) * 64, 0, pol_x);
    }
  }
}

// Attention MMAs of one unit whose stages start at pipeline index iq:
// S = Q K^T into TMEM columns [64, 128), then O = P V^T into [128, 256).
template <int STAGES>
__device__ __forceinline__ bool fwd_att_mma(const FwdProgram& fp, uint8_t* sA, uint64_t* full, uint64_t* empty,
                                            uint64_t* att, uint32_t tmem, long long iq, int au,
                                            volatile int* abort_flag) {
  uint64_t* s_full = att;
  uint64_t* p_full = att + 1;
  uint64_t* o_full = att + 2;
  uint64_t* att_free = att + 3;
  auto st = [&](int j) { return static_cast<int>((iq + j) % STAGES); };
  auto par = [&](int j) { return static_cast<uint32_t>(((iq + j) / STAGES) & 1); };
  if (au >= 1 && !mbar_wait(att_free, (au - 1) & 1, fp.status, abort_flag)) return false;
  for (int j = 0; j < 3; ++j)
    if (!mbar_wait(&full[st(j)], par(j), fp.status, abort_flag)) return false;
  tc_fence_after();
  const uint32_t q0 = smem_u32(sA + st(0) * kATileBytes), q1 = smem_u32(sA + st(1) * kATileBytes);
  const uint32_t kb = smem_u32(sA + st(2) * kATileBytes);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t a = (kk < 4 ? q0 : q1) + (kk & 3) * 32;
    const uint32_t b = kb + (kk >> 2) * (kATileBytes / 2) + (kk & 3) * 32;
    umma_bf16_ss(tmem + kTmemS, sdesc_kmajor_sw128(a), sdesc_kmajor_sw128(b), kAttIdescS, kk > 0 ? 1u : 0u);
  }
  umma_commit(&empty[st(0)]);
  umma_commit(&empty[st(1)]);
  umma_commit(&empty[st(2)]);
  umma_commit(s_full);
  if (!mbar_wait(p_full, au & 1, fp.status, abort_flag)) return false;
  if (!mbar_wait(&full[st(3)], par(3), fp.status, abort_flag)) return false;
  tc_fence_after();
  const uint32_t pa = smem_u32(sA + st(4) * kATileBytes), vb = smem_u32(sA + st(3) * kATileBytes);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    umma_bf16_ss(tmem + kTmemO, sdesc_kmajor_sw128(pa + kk * 32), sdesc_kmajor_sw128(vb + kk * 32), kAttIdescO,
                 kk > 0 ? 1u : 0u);
  umma_commit(&empty[st(3)]);
  umma_commit(&empty[st(4)]);
  umma_commit(o_full);
  return true;
}

// Softmax of one attention unit (128 epilogue threads, thread = row r of the
// query tile: token r / 8, query head g * 8 + r % 8), P into its stage, the
// row's partial output to global scratch.
template <int STAGES>
__device__ __forceinline__ bool fwd_att_softmax(const FwdProgram& fp, uint8_t* sA, uint64_t* full, uint64_t* att,
                                                uint32_t tmem, long long iq, int au, int L, int g, int c,
                                                volatile int* abort_flag) {
  uint64_t* s_full = att;
  uint64_t* p_full = att + 1;
  uint64_t* o_full = att + 2;
  uint64_t* att_free = att + 3;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int et = threadIdx.x - 64;
  const int quarter = warp & 3;
  const int row = quarter * 32 + lane;
  const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
  const int n_rows = fp.qkv.ea.n_rows;
  const int t = row >> 3;
  const int limit = t < fp.n_clean ? L + t + 1 : L + n_rows;  // keys below `limit` are visible
  const int key0 = c * kAttKeys;
  auto st = [&](int j) { return static_cast<int>((iq + j) % STAGES); };
  auto par = [&](int j) { return static_cast<uint32_t>(((iq + j) / STAGES) & 1); };
  bool ok = mbar_wait(s_full, au & 1, fp.status, abort_flag);
  float mx = -INFINITY, lsum = 0.f;
  uint32_t packed[kAttKeys / 2];
  if (ok) {
    tc_fence_after();
    float sc[64];
    tmem_ld64(tmem + lane_off + kTmemS, sc);
    // row max as 8 independent partial maxima (a short dependency chain)
    float m8[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) m8[q] = -INFINITY;
#pragma unroll
    for (int k = 0; k < kAttKeys; ++k)
      if (key0 + k < limit) m8[k & 7] = fmaxf(m8[k & 7], sc[k] * fp.scale_log2);
#pragma unroll
    for (int q = 0; q < 8; ++q) mx = fmaxf(mx, m8[q]);
    float l8[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) l8[q] = 0.f;
#pragma unroll
    for (int k = 0; k < kAttKeys; k += 2) {
      const float p0 = (key0 + k < limit) ? ex2_approx(sc[k] * fp.scale_log2 - mx) : 0.f;
      const float p1 = (key0 + k + 1 < limit) ? ex2_approx(sc[k + 1] * fp.scale_log2 - mx) : 0.f;
      const __half2 ph = __floats2half2_rn(p0, p1);
      const float2 pr = __half22float2(ph);
      l8[(k >> 1) & 7] += pr.x + pr.y;
      packed[k / 2] = *reinterpret_cast<const uint32_t*>(&ph);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) lsum += l8[q];
    ok = mbar_wait(&full[st(4)], par(4), fp.status, abort_flag);  // the P stage is free
  }
  if (ok) {
    uint8_t* prow = sA + st(4) * kATileBytes + row * 128;
#pragma unroll
    for (int cc = 0; cc < 8; ++cc)
      *reinterpret_cast<uint4*>(prow + ((cc ^ (row & 7)) << 4)) =
          make_uint4(packed[cc * 4], packed[cc * 4 + 1], packed[cc * 4 + 2], packed[cc * 4 + 3]);
    // value row d = row to fp16 in place; keys past the cache's valid slots
    // (stale or poisoned, other heads' rows, zero fill) become 0, so that
    // P = 0 there contributes exactly 0
    const int n_valid = L + n_rows - key0;
    ok = mbar_wait(&full[st(3)], par(3), fp.status, abort_flag);
    if (ok) {
      uint8_t* vrow = sA + st(3) * kATileBytes + row * 128;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        // lanes start at different 16-byte chunks of their rows (rows are
        // 128 bytes apart: the same banks)
        const int pos = (i + lane) & 7;
        const int k0 = ((pos ^ (row & 7)) << 3);  // keys k0 .. k0+7 of this 16-byte chunk
        uint4 w = *reinterpret_cast<uint4*>(vrow + (pos << 4));
        uint32_t* wv = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[e]));
          const __half2 hh = __floats2half2_rn(k0 + 2 * e < n_valid ? f.x : 0.f, k0 + 2 * e + 1 < n_valid ? f.y : 0.f);
          wv[e] = *reinterpret_cast<const uint32_t*>(&hh);
        }
        *reinterpret_cast<uint4*>(vrow + (pos << 4)) = w;
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  named_bar_sync(1, 128);
  if (et == 0) mbar_arrive(p_full);
  ok = ok && mbar_wait(o_full, au & 1, fp.status, abort_flag);
  named_bar_sync(1, 128);  // leave together if a wait gave up
  if (*abort_flag) return false;
  tc_fence_after();
  // the unit's partial rows feature-major: each store of the warp covers 32
  // consecutive rows of one feature (128 contiguous bytes)
  const size_t unit = static_cast<size_t>(g * fp.n_chunks_max + c);
  float* dst = fp.apart + unit * 128 * 128 + row;
#pragma unroll 1
  for (int cc = 0; cc < 128; cc += 64) {
    float o[64];
    tmem_ld64(tmem + lane_off + kTmemO + cc, o);
#pragma unroll
    for (int k = 0; k < 64; ++k) __stcg(dst + static_cast<size_t>(cc + k) * 128, o[k]);
  }
  fp.aml[unit * 128 + row] = make_float2(mx, lsum);
  tc_fence_before();
  named_bar_sync(1, 128);
  if (et == 0) mbar_arrive(att_free);
  return true;
}

// Merge of attention rows: CTA b takes the (token t, KV group g) units
// v = b, b + gridDim.x, ... -- 8 rows r = 8 t + (query head within the group)
// -- and warp w their features [32 w, 32 w + 32); lane = (feature quad q,
// row hl), so that one load of the warp covers 4 features x 8 rows (four
// 32-byte pieces).  The rows' weights come first: w_c = 2^(m_c - M), M the
// row's largest chunk max, and l = sum_c w_c l_c; every chunk below
// n_chunks holds a finite partial row (0 where the row sees none of its keys).
constexpr int kMergeMaxChunks = 128;  // 8192 cache slots
__device__ __forceinline__ void fwd_att_merge(const FwdProgram& fp, int L, float* sW) {
  const int lane = threadIdx.x & 31;
  const int et = threadIdx.x - 64;
  const int w = et >> 5;  // 0..3
  const int n_rows = fp.qkv.ea.n_rows;
  const int n_chunks = att_chunks(fp, L);
  float* wts = sW;                      // [8 rows][n_chunks]
  float* inv = sW + 8 * n_chunks;       // [8 rows]
  const int hl = lane & 7, q = lane >> 3;
  for (int v = blockIdx.x; v < n_rows * fp.Hkv; v += gridDim.x) {
    const int t = v / fp.Hkv, g = v % fp.Hkv;
    // weights: thread et takes row et & 7 and chunks et >> 3, + 16, ...
    {
      const int r8 = et & 7;
      const float2* ml = fp.aml + static_cast<size_t>(g) * fp.n_chunks_max * 128 + t * 8 + r8;
      float M = -INFINITY;
      for (int c = et >> 3; c < n_chunks; c += 16) {
        const float2 x = __ldcg(&ml[static_cast<size_t>(c) * 128]);
        if (x.y > 0.f) M = fmaxf(M, x.x);
      }
      // lanes of one row: et, et + 8, ... (the same row in each of the 16 groups of 8)
#pragma unroll
      for (int o = 8; o < 32; o <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
      sW[1152 + et] = M;  // the four warps' maxima, combined below
      named_bar_sync(1, 128);
      M = fmaxf(fmaxf(sW[1152 + r8], sW[1152 + 32 + r8]), fmaxf(sW[1152 + 64 + r8], sW[1152 + 96 + r8]));
      float wl = 0.f;
      for (int c = et >> 3; c < n_chunks; c += 16) {
        const float2 x = __ldcg(&ml[static_cast<size_t>(c) * 128]);
        const float wc = x.y > 0.f ? ex2_approx(x.x - M) : 0.f;
        wts[r8 * n_chunks + c] = wc;
        wl += wc * x.y;
      }
#pragma unroll
      for (int o = 8; o < 32; o <<= 1) wl += __shfl_xor_sync(0xffffffffu, wl, o);
      named_bar_sync(1, 128);
      sW[1152 + et] = wl;
      named_bar_sync(1, 128);
      if (et < 8) {
        const float tot = sW[1152 + et] + sW[1152 + 32 + et] + sW[1152 + 64 + et] + sW[1152 + 96 + et];
        inv[et] = tot > 0.f ? 1.0f / tot : 0.f;
      }
      named_bar_sync(1, 128);
    }
    // features d = 32 w + 4 k + q (k = 0..7) of row hl
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    const float* src = fp.apart + static_cast<size_t>(g) * fp.n_chunks_max * 128 * 128 + t * 8 + hl;
#pragma unroll 2
    for (int c = 0; c < n_chunks; ++c) {
      const float wc = wts[hl * n_chunks + c];
      const float* sc = src + static_cast<size_t>(c) * 128 * 128;
      float f[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) f[k] = __ldcg(sc + static_cast<size_t>(32 * w + 4 * k + q) * 128);
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] += wc * f[k];
    }
    const float iv = inv[hl];
    bf16* out = fp.attn_o + static_cast<size_t>(t) * fp.Hq * 128 + (g * 8 + hl) * 128 + 32 * w + q;
#pragma unroll
    for (int k = 0; k < 8; ++k) out[4 * k] = __float2bfloat16_rn(acc[k] * iv);
    named_bar_sync(1, 128);  // the weights are rewritten by the next unit
  }
}

template <int STAGES>
__global__ void __launch_bounds__(kFwdThreads, 1) fwd_persistent_kernel(const __grid_constant__ FwdProgram fp) {
  constexpr int NT = kFwdNT;
  using S = GemmSmem<NT, STAGES, false>;
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
  uint64_t* att = acce + 2;  // s_full, p_full, o_full, att_free
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  int* sflag = reinterpret_cast<int*>(smem + S::kMisc + 4);
  volatile int* sabort = reinterpret_cast<volatile int*>(smem + S::kMisc + 8);
  const int n_phases = 6 * fp.n_layers;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 2);
      mbar_init(&acce[b], 4);
    }
    for (int k = 0; k < 4; ++k) mbar_init(&att[k], 1);
    *sabort = 0;
    fence_mbar_init();
    for (const ChainPhase* ph : {&fp.qkv, &fp.o, &fp.gu, &fp.down}) {
      tma_prefetch_map(&ph->mapA);
      tma_prefetch_map(&ph->mapB);
    }
    tma_prefetch_map(&fp.gu.mapA2);
    tma_prefetch_map(&fp.mapQ);
    tma_prefetch_map(&fp.mapK);
    tma_prefetch_map(&fp.mapV);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kFwdTmem);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) fwd_load_a<STAGES>(fp, sA, full, empty, sabort);
  } else if (warp == 7) {
    if (lane == 0) fwd_load_b<STAGES>(fp, sA, sB, full, empty, sabort);
  } else if (warp == 1 || warp == kMmaWarp2) {
    if (lane == 0) {
      const int issuer = warp == 1 ? 0 : 1;
      long long i_base = 0;
      int seg = 0, au = 0, L = -1;
      for (int p = 0; p < n_phases; ++p) {
        int layer;
        const int kind = fwd_kind(fp, p, layer);
        if (kind == FK_MERGE) continue;
        if (kind == FK_ATT) {
          if (L < 0) L = fwd_cache_len(fp);
          const int n_units = fp.Hkv * att_chunks(fp, L);
          bool ok = true;
          for (int u = blockIdx.x; u < n_units; u += gridDim.x, i_base += kAttSlots, ++au)
            if (issuer == 0 && !fwd_att_mma<STAGES>(fp, sA, full, empty, att, tmem, i_base, au, sabort)) {
              ok = false;
              break;
            }
          if (!ok) break;
          continue;
        }
        const SkSched sc = chain_sched(fwd_gemm(fp, kind), gridDim.x);
        long long u0, u1;
        chain_range(sc, u0, u1);
        if (!ws_mma_units<NT, STAGES, false>(sA, sB, full, empty, accf, acce, tmem, sc, u0, u1, fp.status, sabort,
                                             issuer, 0, i_base, seg))
          break;
      }
    }
  } else {
    // ------------------------------------------------- epilogue, softmax, merge
    const int et = threadIdx.x - 64;  // 0..127
    griddep_wait();
    // dependents start only once this kernel's own inputs are complete
    if (et == 0) griddep_launch_dependents();
    const int L = fp.qkv.ea.d_len ? *fp.qkv.ea.d_len : fp.qkv.ea.L_static;
    int gseg = 0, au = 0;
    long long i_base = 0;
    bool ok = true;
    for (int p = 0; p < n_phases; ++p) {
      int layer;
      const int kind = fwd_kind(fp, p, layer);
      if (p > 0) {
        if (et == 0) {
          *sflag = ok && wait_counter(fp.bar, p * static_cast<int>(gridDim.x), fp.status, sabort) ? 1 : 0;
          __threadfence();
        }
        named_bar_sync(1, 128);
        ok = *sflag != 0;
        named_bar_sync(1, 128);  // sflag is read before the phase may reuse it
      }
      if (kind == FK_ATT) {
        const int n_chunks = att_chunks(fp, L);
        const int n_units = fp.Hkv * n_chunks;
        for (int u = blockIdx.x; u < n_units; u += gridDim.x, i_base += kAttSlots, ++au)
          if (ok)
            ok = fwd_att_softmax<STAGES>(fp, sA, full, att, tmem, i_base, au, L, u / n_chunks, u % n_chunks,
                                         sabort);
      } else if (kind == FK_MERGE) {
        if (ok) fwd_att_merge(fp, L, sE);
      } else {
        const ChainPhase& ph = fwd_gemm(fp, kind);
        const SkSched sc = chain_sched(ph, gridDim.x);
        long long u0, u1;
        chain_range(sc, u0, u1);
        if (ok) {
          GemmEpi ea = ph.ea;
          if (kind == FK_QKV) {
            ea.kcache += layer * fp.kv_layer;
            ea.vcache += layer * fp.kv_layer;
          }
          if (kind != FK_O && kind != FK_DOWN) ws_rms_factors<NT>(ea, et, sR, sE);
          const int base = fwd_row_base(fp, kind, layer);
          if (kind == FK_QKV)
            ok = ws_epilogue_units<NT, EPI_QKV, false>(sc, u0, u1, base, ea, tmem, accf, acce, sE, sR, nullptr,
                                                       nullptr, sflag, sabort, gseg, L);
          else if (kind == FK_GU)
            ok = ws_epilogue_units<NT, EPI_SWIGLU, false>(sc, u0, u1, base, ea, tmem, accf, acce, sE, sR, nullptr,
                                                          nullptr, sflag, sabort, gseg, 0);
          else
            ok = ws_epilogue_units<NT, EPI_RESID, false>(sc, u0, u1, base, ea, tmem, accf, acce, sE, sR, nullptr,
                                                         nullptr, sflag, sabort, gseg, 0);
        }
        i_base += u1 - u0;
      }
      if (p + 1 < n_phases) {
        // this CTA's phase outputs, plain stores, are read by TMA in other CTAs
        fence_proxy_async_global();
        named_bar_sync(1, 128);
        if (et == 0) {
          __threadfence();
          red_release_gpu_add(fp.bar, 1);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (*sabort) {
    // a wait gave up: let copies already issued land before the CTA's shared
    // memory is released (they complete in microseconds)
    const long long t0 = clock64();
    while (clock64() - t0 < 4000000) {
    }
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kFwdTmem);
  }
  if (threadIdx.x == 0) {
    // every thread of this CTA is past its last barrier wait; the last CTA
    // out zeroes both counters for the next launch
    __threadfence();
    if (atomicAdd(fp.bar + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      fp.bar[0] = 0;
      fp.bar[1] = 0;
      __threadfence();
    }
  }
}

template <int NT, int ST, int EPI, bool FP8 = false>
static cudaError_t launch_one(const CUtensorMap& mapA, const CUtensorMap& mapA2, const CUtensorMap& mapB,
                              const SkSched& sc, int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s) {
  using S = GemmSmem<NT, ST, FP8>;
  auto kern = gemm_ws_kernel<NT, ST, EPI, FP8>;
  // function attributes are per device: set once on each device that launches
  static bool attr_set[64] = {};
  int dev_ = 0;
  if (cudaGetDevice(&dev_) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev_ < 0 || dev_ >= 64 || !attr_set[dev_]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal);
    if (e != cudaSuccess) return e;
    if (dev_ >= 0 && dev_ < 64) attr_set[dev_] = true;
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

template <int NT, int ST, int EPI, bool FP8 = false>
static cudaError_t launch_cl(const CUtensorMap& mapA, const CUtensorMap& mapB, int n_tiles, int kb, int S,
                             int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s) {
  using Sm = ClSmem<NT, ST, FP8>;
  auto kern = gemm_cl_kernel<NT, ST, EPI, FP8>;
  // function attributes are per device: set once on each device that launches
  static bool attr_set[64] = {};
  int dev_ = 0;
  if (cudaGetDevice(&dev_) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev_ < 0 || dev_ >= 64 || !attr_set[dev_]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sm::kTotal);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    if (dev_ >= 0 && dev_ < 64) attr_set[dev_] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_tiles * S);
  cfg.blockDim = dim3(kWsThreads);
  cfg.dynamicSmemBytes = Sm::kTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = S;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, mapA, mapB, kb, S, a_row_base, ea);
}

cudaError_t launch_gemm_cl(int NT, const CUtensorMap& mapA, const CUtensorMap& mapB, int n_tiles, int kb, int S,
                           int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s, int stages) {
  if (S < 2 || S > 16 || NT != 16) return cudaErrorInvalidValue;
  if (stages == 5) {
    if (ea.epi == EPI_QKV) return launch_cl<16, 5, EPI_QKV>(mapA, mapB, n_tiles, kb, S, a_row_base, ea, pdl, s);
    if (ea.epi == EPI_RESID) return launch_cl<16, 5, EPI_RESID>(mapA, mapB, n_tiles, kb, S, a_row_base, ea, pdl, s);
  }
  if (stages == 10) {
    if (ea.epi == EPI_QKV) return launch_cl<16, 10, EPI_QKV>(mapA, mapB, n_tiles, kb, S, a_row_base, ea, pdl, s);
    if (ea.epi == EPI_RESID) return launch_cl<16, 10, EPI_RESID>(mapA, mapB, n_tiles, kb, S, a_row_base, ea, pdl, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_cl_fp8(const CUtensorMap& mapA, int n_tiles, int kb, int S, int a_row_base, const GemmEpi& ea,
                               bool pdl, cudaStream_t s, int stages) {
  if (S < 2 || S > 16 || (kb + S - 1) / S > kMaxFp8Blocks) return cudaErrorInvalidValue;
  if (stages == 5) {
    if (ea.epi == EPI_QKV) return launch_cl<16, 5, EPI_QKV, true>(mapA, mapA, n_tiles, kb, S, a_row_base, ea, pdl, s);
    if (ea.epi == EPI_RESID)
      return launch_cl<16, 5, EPI_RESID, true>(mapA, mapA, n_tiles, kb, S, a_row_base, ea, pdl, s);
  }
  if (stages == 10) {
    if (ea.epi == EPI_QKV)
      return launch_cl<16, 10, EPI_QKV, true>(mapA, mapA, n_tiles, kb, S, a_row_base, ea, pdl, s);
    if (ea.epi == EPI_RESID)
      return launch_cl<16, 10, EPI_RESID, true>(mapA, mapA, n_tiles, kb, S, a_row_base, ea, pdl, s);
  }
  return cudaErrorInvalidValue;
}

// Stream-K W8A8 kernel: every CTA's range must need at most kMaxFp8Blocks
// activation code blocks (a range that crosses a tile boundary needs all kb).
cudaError_t launch_gemm_ws_fp8(const CUtensorMap& mapA, const CUtensorMap& mapA2, int n_tiles, int kb, int P,
                               int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s) {
  if (kb > kMaxFp8Blocks) return cudaErrorInvalidValue;
  SkSched sc{n_tiles, kb, P};
  if (ea.epi == EPI_SWIGLU) return launch_one<16, 10, EPI_SWIGLU, true>(mapA, mapA2, mapA, sc, a_row_base, ea, pdl, s);
  if (ea.epi == EPI_RESID) return launch_one<16, 10, EPI_RESID, true>(mapA, mapA2, mapA, sc, a_row_base, ea, pdl, s);
  if (ea.epi == EPI_QKV) return launch_one<16, 10, EPI_QKV, true>(mapA, mapA2, mapA, sc, a_row_base, ea, pdl, s);
  return cudaErrorInvalidValue;
}

// Clusters of S CTAs of the cluster split-K kernel that can be resident at
// once (0: that cluster size cannot be launched).
template <int ST, bool FP8 = false>
static int cl_max_clusters(int epi, int S) {
  using Sm = ClSmem<16, ST, FP8>;
  auto kern = epi == EPI_QKV ? gemm_cl_kernel<16, ST, EPI_QKV, FP8> : gemm_cl_kernel<16, ST, EPI_RESID, FP8>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sm::kTotal) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S * 16);
  cfg.blockDim = dim3(kWsThreads);
  cfg.dynamicSmemBytes = Sm::kTotal;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = S;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int gemm_cl_max_clusters(int epi, int S, int stages) {
  return stages == 10 ? cl_max_clusters<10>(epi, S) : cl_max_clusters<5>(epi, S);
}

int gemm_cl_max_clusters_fp8(int epi, int S, int stages) {
  return stages == 10 ? cl_max_clusters<10, true>(epi, S) : cl_max_clusters<5, true>(epi, S);
}

size_t gemm_ws_part_bytes(int NT, int P) { return static_cast<size_t>(P) * NT * 128 * sizeof(float); }

cudaError_t launch_gemm_ws(int NT, const CUtensorMap& mapA, const CUtensorMap& mapA2, const CUtensorMap& mapB,
                           int n_tiles, int kb, int P, int a_row_base, const GemmEpi& ea, bool pdl, cudaStream_t s,
                           int stages) {
  SkSched sc{n_tiles, kb, P};
#define DVLM_GEMM_CASE(nt, st)                                                                         \
  if (NT == nt && stages == st) {                                                                      \
    switch (ea.epi) {                                                                                  \
      case EPI_QKV: return launch_one<nt, st, EPI_QKV>(mapA, mapA2, mapB, sc, a_row_base, ea, pdl, s);       \
      case EPI_RESID: return launch_one<nt, st, EPI_RESID>(mapA, mapA2, mapB, sc, a_row_base, ea, pdl, s);   \
      case EPI_SWIGLU: return launch_one<nt, st, EPI_SWIGLU>(mapA, mapA2, mapB, sc, a_row_base, ea, pdl, s); \
    }                                                                                                  \
  }
  DVLM_GEMM_CASE(16, 5)
  DVLM_GEMM_CASE(16, 10)
  DVLM_GEMM_CASE(32, 4)
#undef DVLM_GEMM_CASE
  return cudaErrorInvalidValue;
}

static int fwd_cap[64] = {};  // resident CTAs per device (0: not yet queried)

int fwd_persistent_max_ctas() {
  using S = GemmSmem<kFwdNT, kFwdStages, false>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (fwd_cap[dev] == 0) {
    auto kern = fwd_persistent_kernel<kFwdStages>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal) != cudaSuccess) return 0;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFwdThreads, S::kTotal) != cudaSuccess)
      return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    fwd_cap[dev] = per_sm * sms;
  }
  return fwd_cap[dev];
}

size_t fwd_attn_scratch_bytes(int Hkv, int Lmax) {
  const size_t n_chunks = (static_cast<size_t>(Lmax) + kAttKeys - 1) / kAttKeys;
  const size_t part = static_cast<size_t>(Hkv) * n_chunks * 128 * 128 * 4;
  const size_t ml = static_cast<size_t>(Hkv) * n_chunks * 128 * 8;
  return (part + 255) / 256 * 256 + (ml + 255) / 256 * 256;
}

cudaError_t launch_fwd_persistent(const FwdProgram& fp, int P, bool pdl, cudaStream_t s) {
  using S = GemmSmem<kFwdNT, kFwdStages, false>;
  if (fp.n_layers < 1 || P < 1 || !fp.bar || !fp.status || !fp.apart || !fp.aml || !fp.attn_o)
    return cudaErrorInvalidValue;
  if (fp.Hq != 8 * fp.Hkv || fp.n_chunks_max < (fp.Lmax + kAttKeys - 1) / kAttKeys ||
      fp.n_chunks_max > kMergeMaxChunks)
    return cudaErrorInvalidValue;
  for (const ChainPhase* ph : {&fp.qkv, &fp.o, &fp.gu, &fp.down}) {
    if (ph->n_tiles < 1 || ph->kb < 1 || ph->ea.n_rows < 1 || ph->ea.n_rows > kFwdNT || !ph->ea.part ||
        !ph->ea.cnt || ph->ea.status != fp.status)
      return cudaErrorInvalidValue;
  }
  if (fp.qkv.ea.epi != EPI_QKV || fp.o.ea.epi != EPI_RESID || fp.gu.ea.epi != EPI_SWIGLU ||
      fp.down.ea.epi != EPI_RESID)
    return cudaErrorInvalidValue;
  // every CTA must be resident at once: the phases meet at grid barriers
  const int cap = fwd_persistent_max_ctas();
  if (cap < 1) return cudaErrorInvalidConfiguration;
  if (P > cap) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P);
  cfg.blockDim = dim3(kFwdThreads);
  cfg.dynamicSmemBytes = S::kTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fwd_persistent_kernel<kFwdStages>, fp);
}

}  // namespace dvlm
