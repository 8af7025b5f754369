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
  static constexpr int kMisc = kBar + (2 * STAGES + 5) * 8;
  static constexpr int kTotal = kMisc + 64 + 1024;  // + alignment slack
};

// Per-row scale of an E4M3 weight tile row (absolute weight row index).
__device__ __forceinline__ float fp8_row_scale(const GemmEpi& ea, bool split, int a_row_base, int T, int row) {
  if (split) return row < 64 ? ea.wscale[a_row_base + T * 64 + row] : ea.wscale2[a_row_base + T * 64 + row - 64];
  return ea.wscale[a_row_base + T * 128 + row];
}

// RMSNorm factors of the NT input rows from the producers' per-tile sums of
// squares (ssq_in [n_ssq][NT]), run by the 128 epilogue threads: 128 / NT
// partial sums per row with independent loads, then one thread per row adds
// the partials in order.  sPart: 128 floats of scratch.
template <int NT>
__device__ __forceinline__ void ws_rms_factors(const GemmEpi& ea, int et, float* sR, float* sPart) {
  constexpr int G = 128 / NT;
  const int t = et % NT, g = et / NT;
  float s = 0.f;
  for (int q = g; q < ea.n_ssq; q += G) s += __ldcg(&ea.ssq_in[q * NT + t]);
  sPart[g * NT + t] = s;
  named_bar_sync(1, 128);
  if (et < NT) {
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < G; ++k) tot += sPart[k * NT + et];
    sR[et] = 1.0f / sqrtf(tot * ea.inv_h + ea.eps);
  }
  named_bar_sync(1, 128);
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
    if (EPI == EPI_QKV && et < NT) {
      float s2 = 0.f;
      for (int p = 0; p < ea.n_ssq; ++p) s2 += ea.ssq_in[p * NT + et];
      sR[et] = 1.0f / sqrtf(s2 * ea.inv_h + ea.eps);
    }
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
// Persistent GEMM chain.  The products that follow a layer's attention --
// O-projection (+ residual), gate/up (SwiGLU), down (+ residual) -- and the
// next layer's QKV run as consecutive stream-K phases of one launch on every
// SM, instead of one kernel each.  A phase reads what the previous phase's
// epilogues wrote (all CTAs), so a grid barrier separates the phases: every
// CTA bumps a counter after its phase epilogue, and phase p's inputs are
// ready once the counter reaches p * P.  The weight stream never waits for
// it: the A loader runs through the phases back to back, so while the last
// split tiles of one phase are being reduced and finished, the next phase's
// weight tiles already fill the pipeline stages.  Only the activation tiles
// (2 KB a stage, L2-resident) wait for the barrier, issued by a loader warp
// of their own that polls it.  One A loader arrival per stage arms the
// stage's full barrier with A + B bytes (a B copy may complete before that
// arrival; the phase still needs the arrival).
//
// Roles (256 threads): warp 0 A loader, warps 1 and 6 MMA issuers, warps
// 2..5 epilogue, warp 7 B loader.  All P CTAs must be resident together
// (one per SM; the launcher checks the occupancy), and every wait is
// bounded: a CTA that gives up records DVLM_ERR_TIMEOUT and still arrives
// at the remaining barriers, so the others do not wait on it.
constexpr int kChainThreads = 256;
constexpr int kChainStages = 12;
constexpr int kChainNT = 16;

// A phase's stream-K schedule: its units over min(P, units) CTAs (a CTA with
// an empty range between the CTAs of a split tile would be counted as one of
// its contributors); CTAs past those have no units in the phase.
__device__ __forceinline__ SkSched chain_sched(const ChainPhase& ph, int P) {
  const long long units = static_cast<long long>(ph.n_tiles) * ph.kb;
  return SkSched{ph.n_tiles, ph.kb, static_cast<int>(units < P ? units : P)};
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
__device__ __forceinline__ void chain_load_a(const ChainArgs& ca, uint8_t* sA, uint64_t* full, uint64_t* empty,
                                             volatile int* abort_flag) {
  constexpr int B_BYTES = kChainNT * 128;
  const uint64_t pol_w = l2_policy_evict_first();
  long long i = 0;
  for (int p = 0; p < ca.n_phases; ++p) {
    const ChainPhase& ph = ca.ph[p];
    const SkSched sc = chain_sched(ph, ca.P);
    long long u0, u1;
    chain_range(sc, u0, u1);
    const bool split = ph.ea.epi == EPI_SWIGLU;
    for (long long u = u0; u < u1; ++u, ++i) {
      const int s = static_cast<int>(i % STAGES);
      if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, ca.status, abort_flag)) return;
      mbar_arrive_expect_tx(&full[s], kATileBytes + B_BYTES);
      const int T = static_cast<int>(u / sc.kb), kk = static_cast<int>(u % sc.kb);
      if (split) {
        tma_load_2d(sA + s * kATileBytes, &ph.mapA, &full[s], kk * 64, ph.a_row_base + T * 64, pol_w);
        tma_load_2d(sA + s * kATileBytes + kATileBytes / 2, &ph.mapA2, &full[s], kk * 64, ph.a_row_base + T * 64,
                    pol_w);
      } else {
        tma_load_2d(sA + s * kATileBytes, &ph.mapA, &full[s], kk * 64, ph.a_row_base + T * 128, pol_w);
      }
    }
  }
}

template <int STAGES>
__device__ __forceinline__ void chain_load_b(const ChainArgs& ca, uint8_t* sB, uint64_t* full, uint64_t* empty,
                                             volatile int* abort_flag) {
  constexpr int B_BYTES = kChainNT * 128;
  const uint64_t pol_x = l2_policy_evict_last();
  long long i = 0;
  for (int p = 0; p < ca.n_phases; ++p) {
    // inputs of phase p: the kernel before this one (p = 0), else every CTA's phase p-1
    if (p == 0)
      griddep_wait();
    else if (!wait_counter(ca.bar, p * ca.P, ca.status, abort_flag))
      return;
    fence_proxy_async_global();
    const ChainPhase& ph = ca.ph[p];
    const SkSched sc = chain_sched(ph, ca.P);
    long long u0, u1;
    chain_range(sc, u0, u1);
    for (long long u = u0; u < u1; ++u, ++i) {
      const int s = static_cast<int>(i % STAGES);
      if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, ca.status, abort_flag)) return;
      tma_load_2d(sB + s * B_BYTES, &ph.mapB, &full[s], static_cast<int>(u % sc.kb) * 64, 0, pol_x);
    }
  }
}

template <int STAGES>
__global__ void __launch_bounds__(kChainThreads, 1) gemm_chain_kernel(const __grid_constant__ ChainArgs ca) {
  constexpr int NT = kChainNT;
  using S = GemmSmem<NT, STAGES, false>;
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
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 2);
      mbar_init(&acce[b], 4);
    }
    *sabort = 0;
    fence_mbar_init();
    for (int p = 0; p < ca.n_phases; ++p) {
      tma_prefetch_map(&ca.ph[p].mapA);
      tma_prefetch_map(&ca.ph[p].mapB);
      if (ca.ph[p].ea.epi == EPI_SWIGLU) tma_prefetch_map(&ca.ph[p].mapA2);
    }
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
    if (lane == 0) chain_load_a<STAGES>(ca, sA, full, empty, sabort);
  } else if (warp == 7) {
    if (lane == 0) chain_load_b<STAGES>(ca, sB, full, empty, sabort);
  } else if (warp == 1 || warp == kMmaWarp2) {
    if (lane == 0) {
      long long i_base = 0;
      int seg = 0;
      for (int p = 0; p < ca.n_phases; ++p) {
        const SkSched sc = chain_sched(ca.ph[p], ca.P);
        long long u0, u1;
        chain_range(sc, u0, u1);
        if (!ws_mma_units<NT, STAGES, false>(sA, sB, full, empty, accf, acce, tmem, sc, u0, u1, ca.status, sabort,
                                             warp == 1 ? 0 : 1, 0, i_base, seg))
          break;
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int et = threadIdx.x - 64;  // 0..127
    griddep_wait();
    // dependents start only once this kernel's own inputs are complete
    if (et == 0) griddep_launch_dependents();
    int gseg = 0;
    bool ok = true;
    for (int p = 0; p < ca.n_phases; ++p) {
      const ChainPhase& ph = ca.ph[p];
      const GemmEpi& ea = ph.ea;
      if (p > 0) {
        if (et == 0) {
          *sflag = ok && wait_counter(ca.bar, p * ca.P, ca.status, sabort) ? 1 : 0;
          __threadfence();
        }
        named_bar_sync(1, 128);
        ok = *sflag != 0;
        named_bar_sync(1, 128);  // sflag is read before the phase may reuse it
      }
      if (ok) {
        if (ea.epi != EPI_RESID) ws_rms_factors<NT>(ea, et, sR, sE);
        const SkSched sc = chain_sched(ph, ca.P);
        long long u0, u1;
        chain_range(sc, u0, u1);
        if (ea.epi == EPI_QKV)
          ok = ws_epilogue_units<NT, EPI_QKV, false>(sc, u0, u1, ph.a_row_base, ea, tmem, accf, acce, sE, sR,
                                                     nullptr, nullptr, sflag, sabort, gseg,
                                                     ea.d_len ? *ea.d_len : ea.L_static);
        else if (ea.epi == EPI_SWIGLU)
          ok = ws_epilogue_units<NT, EPI_SWIGLU, false>(sc, u0, u1, ph.a_row_base, ea, tmem, accf, acce, sE, sR,
                                                        nullptr, nullptr, sflag, sabort, gseg, 0);
        else
          ok = ws_epilogue_units<NT, EPI_RESID, false>(sc, u0, u1, ph.a_row_base, ea, tmem, accf, acce, sE, sR,
                                                       nullptr, nullptr, sflag, sabort, gseg, 0);
      }
      if (p + 1 < ca.n_phases) {
        // this CTA's phase outputs, plain stores, are read by TMA in other CTAs
        fence_proxy_async_global();
        named_bar_sync(1, 128);
        if (et == 0) {
          __threadfence();
          red_release_gpu_add(ca.bar, 1);
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
    tmem_dealloc(tmem, TMC);
  }
  if (threadIdx.x == 0) {
    // every thread of this CTA is past its last barrier wait; the last CTA
    // out zeroes both counters for the next launch
    __threadfence();
    if (atomicAdd(ca.bar + 1, 1) == static_cast<int>(gridDim.x) - 1) {
      ca.bar[0] = 0;
      ca.bar[1] = 0;
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

static int chain_cap[64] = {};  // resident CTAs per device (0: not yet queried)

int gemm_chain_max_ctas() {
  using S = GemmSmem<kChainNT, kChainStages, false>;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (chain_cap[dev] == 0) {
    auto kern = gemm_chain_kernel<kChainStages>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kTotal) != cudaSuccess) return 0;
    int per_sm = 0, sms = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kChainThreads, S::kTotal) != cudaSuccess)
      return 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    chain_cap[dev] = per_sm * sms;
  }
  return chain_cap[dev];
}

cudaError_t launch_gemm_chain(const ChainArgs& ca, bool pdl, cudaStream_t s) {
  using S = GemmSmem<kChainNT, kChainStages, false>;
  if (ca.n_phases < 1 || ca.n_phases > kMaxChainPhases || ca.P < 1 || !ca.bar || !ca.status)
    return cudaErrorInvalidValue;
  for (int p = 0; p < ca.n_phases; ++p) {
    const ChainPhase& ph = ca.ph[p];
    const int epi = ph.ea.epi;
    if ((epi != EPI_QKV && epi != EPI_RESID && epi != EPI_SWIGLU) || ph.n_tiles < 1 || ph.kb < 1 ||
        ph.ea.n_rows < 1 || ph.ea.n_rows > kChainNT || !ph.ea.part || !ph.ea.cnt || ph.ea.status != ca.status)
      return cudaErrorInvalidValue;
  }
  // every CTA must be resident at once: the phases meet at grid barriers
  const int cap = gemm_chain_max_ctas();
  if (cap < 1) return cudaErrorInvalidConfiguration;
  if (ca.P > cap) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ca.P);
  cfg.blockDim = dim3(kChainThreads);
  cfg.dynamicSmemBytes = S::kTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_chain_kernel<kChainStages>, ca);
}

}  // namespace dvlm
