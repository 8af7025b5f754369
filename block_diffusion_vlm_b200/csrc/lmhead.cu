// Fused LM head + top-1 confidence + argmax + threshold commit (+ certificate).
//
// logits[v, t] = s_t * sum_k W[v, k] h[t, k] are produced 128 vocabulary rows
// at a time in TMEM by tcgen05 UMMAs (W streamed once from HBM through TMA)
// and folded straight into a running (max m, sum of exp(l - m), argmax) per
// token; logits never reach memory.  p1 = 1 / sum exp(l - max) is the top-1
// softmax probability [Look Only When Needed, method step (1)]; the argmax is
// the lowest id among equal maxima.  The last CTA to finish merges all
// per-CTA records in CTA order (deterministic) and applies the commit rule.
#include "finalize.cuh"
#include "mainloop.cuh"

namespace dvlm {

template <int NT>
struct LmCfg {
  // Bytes in flight per SM bound a streaming kernel at batch 1: one CTA per
  // SM keeps 160-180 KB of weight tiles in flight for the narrow row counts.
  static constexpr int STAGES = NT <= 16 ? 10 : (NT <= 32 ? 9 : 4);
  static constexpr int TPT = 128 / NT;     // scan threads per token
  static constexpr int SROW = 128 + TPT;   // padded row of the transposed tile (bank-conflict free)
  static constexpr int kA = 0;
  static constexpr int kB = kA + STAGES * kATileBytes;
  static constexpr int kT = kB + STAGES * NT * 128;
  static constexpr int kRec = kT + NT * SROW * 4;
  static constexpr int kFin = kRec + 128 * 16;
  static constexpr int kBar = kFin + ((static_cast<int>(sizeof(FinalizeSmem)) + 15) / 16) * 16;
  static constexpr int kMisc = kBar + (2 * STAGES + 4) * 8;
  static constexpr int kTotal = kMisc + 64 + 1024;
};

struct Stat {
  float m, s;
  int idx;
};

__device__ __forceinline__ void stat_push(Stat& st, float l, int v) {
  if (l > st.m) {
    st.s = st.s * expf(st.m - l) + 1.0f;
    st.m = l;
    st.idx = v;
  } else {
    st.s += expf(l - st.m);
  }
}
// (m1,s1,i1) <- (m1,s1,i1) (+) (m2,s2,i2); empty records have s == 0.
__device__ __forceinline__ void stat_merge(Stat& a, const Stat& b) {
  if (b.s == 0.0f) return;
  if (a.s == 0.0f) {
    a = b;
    return;
  }
  if (b.m > a.m) {
    a.s = a.s * expf(a.m - b.m) + b.s;
    a.m = b.m;
    a.idx = b.idx;
  } else if (b.m == a.m) {
    a.s += b.s;
    a.idx = b.idx < a.idx ? b.idx : a.idx;
  } else {
    a.s += b.s * expf(b.m - a.m);
  }
}

template <int NT, int STAGES>
__global__ void __launch_bounds__(kWsThreads, 1)
    lmhead_kernel(const __grid_constant__ CUtensorMap mapW, const __grid_constant__ CUtensorMap mapH,
                  const SkSched sc, const LmArgs a) {
  using C = LmCfg<NT>;
  constexpr int TMC = tmem_cols_for<NT>();
  constexpr int TPT = C::TPT, SROW = C::SROW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align1024(smem_raw);
  uint8_t* sA = smem + C::kA;
  uint8_t* sB = smem + C::kB;
  float* sT = reinterpret_cast<float*>(smem + C::kT);  // [NT][SROW] logits, token-major
  float4* sRec = reinterpret_cast<float4*>(smem + C::kRec);
  FinalizeSmem& fs = *reinterpret_cast<FinalizeSmem*>(smem + C::kFin);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBar);
  uint64_t* empty = full + STAGES;
  uint64_t* accf = empty + STAGES;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMisc);
  int* sflag = reinterpret_cast<int*>(smem + C::kMisc + 4);
  volatile int* sabort = reinterpret_cast<volatile int*>(smem + C::kMisc + 8);
  int* slast = reinterpret_cast<int*>(smem + C::kMisc + 12);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = sc.P;
  const long long u0 = sc.begin(blockIdx.x), u1 = sc.begin(blockIdx.x + 1);

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
    tma_prefetch_map(&mapW);
    tma_prefetch_map(&mapH);
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
      ws_producer<NT, STAGES, false>(&mapW, &mapW, &mapH, sA, sB, full, empty, sc, u0, u1, 0, 0, a.status, sabort);
  } else if (warp == 1 || warp == kMmaWarp2) {
    if (lane == 0 && u1 > u0)
      ws_mma<NT, STAGES>(sA, sB, full, empty, accf, acce, tmem, sc, u0, u1, a.status, sabort, warp == 1 ? 0 : 1);
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64;
    const int tok = et / TPT, sub = et % TPT;
    auto bar = [] { named_bar_sync(1, 128); };
    griddep_wait();
    // Dependents may start only once this kernel's own inputs are complete,
    // so at most two kernels of the chain overlap (see ptx.cuh).
    if (et == 0) griddep_launch_dependents();
    float rt = 1.0f;  // final RMSNorm factor of this thread's token
    if (a.ssq_in) {
      float s = 0.f;
      for (int p = 0; p < a.n_ssq; ++p) s += a.ssq_in[p * NT + tok];
      rt = 1.0f / sqrtf(s * a.inv_h + a.eps);
    }
    Stat run{-INFINITY, 0.0f, 0x7fffffff};
    auto scan = [&](int T, Stat& st) {
#pragma unroll 4
      for (int i = 0; i < NT; ++i) {
        const int r = sub + TPT * i;
        const int v = T * 128 + r;
        if (v < a.V) stat_push(st, sT[tok * SROW + r] * rt, v);
      }
    };
    // Combine the TPT per-thread records of each token in sub order.
    auto combine = [&](Stat st) -> Stat {
      sRec[et] = make_float4(st.m, st.s, __int_as_float(st.idx), 0.f);
      bar();
      Stat out{-INFINITY, 0.0f, 0x7fffffff};
      if (sub == 0) {
        for (int k = 0; k < TPT; ++k) {
          const float4 f = sRec[tok * TPT + k];
          stat_merge(out, Stat{f.x, f.y, __float_as_int(f.z)});
        }
      }
      bar();
      return out;
    };
    // A vocabulary tile split over CTAs pf < ... < pl is finished by pf, which
    // streams the tile's first k blocks as its last segment; the others
    // stream their parts first and leave fp32 partial logits in global
    // scratch, counted on cnt[T].  pf fetches them while its own last
    // segment is still in the mainloop, adds them in CTA order and scans the
    // tile into its running record like any whole tile.
    int seg = 0;
    bool ok = true;
    for (long long u = u0; u < u1; ++seg) {
      const int T = static_cast<int>(u / sc.kb);
      const long long t_begin = static_cast<long long>(T) * sc.kb, t_end = t_begin + sc.kb;
      const long long seg_end = t_end < u1 ? t_end : u1;
      const int b = seg & 1;
      const bool whole = (u == t_begin) && (seg_end == t_end);
      const bool finisher = !whole && (u == t_begin);
      float o[NT];  // the other CTAs' partial logits of row et (finisher)
      if (finisher) {
        const int pl = sc.cta_of(t_end - 1);
        if (et == 0) {
          const bool got = wait_counter(&a.cnt[T], pl - static_cast<int>(blockIdx.x), a.status, sabort);
          if (got) a.cnt[T] = 0;  // every part is counted: zero again for the next launch
          *sflag = got ? 1 : 0;
        }
        bar();
        if (!*sflag) {
          ok = false;
          break;
        }
        __threadfence();
#pragma unroll
        for (int t = 0; t < NT; ++t) o[t] = 0.f;
        // the other CTAs' partials in CTA order, kQ sources' loads in flight
        constexpr int kQ = NT <= 32 ? 2 : 1;
        for (int p0 = static_cast<int>(blockIdx.x) + 1; p0 <= pl; p0 += kQ) {
          float q2[kQ][NT];
#pragma unroll
          for (int q = 0; q < kQ; ++q) {
            const float* src = a.part + static_cast<size_t>(p0 + q <= pl ? p0 + q : p0) * NT * 128;
#pragma unroll
            for (int t = 0; t < NT; ++t) q2[q][t] = __ldcg(&src[t * 128 + et]);
          }
#pragma unroll
          for (int q = 0; q < kQ; ++q)
            if (p0 + q <= pl) {
#pragma unroll
              for (int t = 0; t < NT; ++t) o[t] += q2[q][t];
            }
        }
      }
      mbar_wait(&accf[b], (seg >> 1) & 1, a.status, sabort);
      bar();
      if (*sabort) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < NT; c += 16) {
        float acc[16];
        ws_load_acc16<NT>(tmem, b, quarter, c, acc, seg_end - u >= 2);
#pragma unroll
        for (int k = 0; k < 16; ++k) sT[(c + k) * SROW + row] = acc[k];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acce[b]);
      bar();
      if (!whole && !finisher) {
        // tail or middle part of a tile finished by another CTA
        float* mine = a.part + static_cast<size_t>(blockIdx.x) * NT * 128;
#pragma unroll
        for (int t = 0; t < NT; ++t) __stcg(&mine[t * 128 + et], sT[t * SROW + et]);
        __threadfence();
        bar();
        if (et == 0) red_release_gpu_add(&a.cnt[T], 1);
      } else {
        if (finisher) {
#pragma unroll
          for (int t = 0; t < NT; ++t) sT[t * SROW + et] += o[t];
          bar();
        }
        scan(T, run);
      }
      bar();  // sT is rewritten by the next segment
      u = seg_end;
    }
    if (ok) {
      const Stat mine = combine(run);
      if (sub == 0) {
        float4* dst = reinterpret_cast<float4*>(a.rec) + static_cast<size_t>(blockIdx.x) * NT + tok;
        __stcg(dst, make_float4(mine.m, mine.s, __int_as_float(mine.idx), 0.f));
      }
      __threadfence();
      bar();
      if (et == 0) {
        const int old = atomicAdd(a.done, 1);
        *slast = (old == P - 1) ? 1 : 0;
      }
      bar();
      if (*slast) {
        __threadfence();
        // The last CTA merges every CTA's record of each token in CTA order;
        // a thread's records are fetched in batches of 16 loads in flight.
        Stat st{-INFINITY, 0.0f, 0x7fffffff};
        const float4* rec = reinterpret_cast<const float4*>(a.rec);
        constexpr int kBatch = 16;
        for (int p0 = sub; p0 < P; p0 += TPT * kBatch) {
          float4 f[kBatch];
#pragma unroll
          for (int q = 0; q < kBatch; ++q) {
            const int p = p0 + TPT * q;
            f[q] = p < P ? __ldcg(&rec[static_cast<size_t>(p) * NT + tok]) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int q = 0; q < kBatch; ++q)
            if (p0 + TPT * q < P) stat_merge(st, Stat{f[q].x, f[q].y, __float_as_int(f[q].z)});
        }
        const Stat fin = combine(st);
        if (sub == 0 && tok < 128) {
          fs.p1[tok] = fin.s > 0.f ? 1.0f / fin.s : 0.0f;
          fs.id[tok] = fin.idx;
        }
        bar();
        if (et == 0) *a.done = 0;
        finalize_rows(et, a, fs, bar);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, TMC);
  }
}

size_t lmhead_scratch_bytes(int NT, int P, int n_tiles) {
  size_t part = static_cast<size_t>(P) * NT * 128 * 4;
  size_t rec = static_cast<size_t>(P) * NT * 16;
  size_t ints = (static_cast<size_t>(n_tiles) + 1) * 4;
  return part + rec + ints + 256;
}

template <int NT>
static cudaError_t lm_launch(const CUtensorMap& mapW, const CUtensorMap& mapH, const SkSched& sc, const LmArgs& a,
                             bool pdl, cudaStream_t s) {
  using C = LmCfg<NT>;
  auto kern = lmhead_kernel<NT, C::STAGES>;
  // function attributes are per device: set once on each device that launches
  static bool attr_set[64] = {};
  int dev_ = 0;
  if (cudaGetDevice(&dev_) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev_ < 0 || dev_ >= 64 || !attr_set[dev_]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kTotal);
    if (e != cudaSuccess) return e;
    if (dev_ >= 0 && dev_ < 64) attr_set[dev_] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(sc.P);
  cfg.blockDim = dim3(kWsThreads);
  cfg.dynamicSmemBytes = C::kTotal;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, mapW, mapH, sc, a);
}

cudaError_t launch_lmhead(int NT, const CUtensorMap& mapW, const CUtensorMap& mapH, int n_tiles, int kb, int P,
                          const LmArgs& a, bool pdl, cudaStream_t s) {
  SkSched sc{n_tiles, kb, P};
  switch (NT) {
    case 16: return lm_launch<16>(mapW, mapH, sc, a, pdl, s);
    case 32: return lm_launch<32>(mapW, mapH, sc, a, pdl, s);
    case 64: return lm_launch<64>(mapW, mapH, sc, a, pdl, s);
    case 128: return lm_launch<128>(mapW, mapH, sc, a, pdl, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dvlm
