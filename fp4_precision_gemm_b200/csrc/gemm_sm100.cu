// Block-scaled low-precision GEMM on the sm_100a tensor cores:
//   C[M x N] (BF16) = A[M x K] . B[N x K]^T with both operands K-major codes.
//
// "Can you explain the role of FP8 precision in DeepSeek-V3 training":
//   "Mixed-precision framework" - the compute-heavy GEMMs run in FP8 (fprop, dgrad, wgrad);
//   "Fine-grained quantization" - 1x128 activation tiles and 128x128 weight blocks;
//   "Increased accumulation precision" - partial results are promoted to FP32 at fixed
//   intervals.  Here the interval is one 128-element K chunk: the tensor cores form the
//   chunk's E4M3 partial product in a TMEM buffer, and CUDA cores add it, times the chunk's
//   two scales, into an FP32 accumulator held in registers.
// "Accelerating FP8 training performance with the NVIDIA NeMo framework": MXFP8 (block
//   processing in the Blackwell tensor cores: E8M0 scales applied by the MMA itself) and the
//   per-tensor recipe.
// "NVIDIA developed a method to train neural networks in 4-bit precision": NVFP4 (E2M1 with
//   per-16 E4M3 scales applied by the MMA, per-tensor FP32 scales in the epilogue).
//
// Kernel structure (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 8     TMA producer: A/B stages (128 bytes of K, 128B-swizzled), scale stages;
//   warp 9     TMEM allocator and the single MMA-issuing thread;
//   warps 0-7  epilogue: warp w reads TMEM lanes 32*(w%4).. (its 32 output rows) and
//              columns 128*(w/4).. of the tile.
// Blockwise: two 256-column TMEM partial buffers alternate per K chunk, so the MMAs of chunk
// k+1 run while the epilogue warps promote chunk k; the 128 FP32 accumulators per thread
// stay in registers for the whole tile.  Other recipes accumulate in one TMEM buffer and
// the epilogue drains it once per tile.
// Every wait is bounded: a wait that runs out records a timeout in the device status word,
// raises the CTA's abort flag and the roles wind down (waiting, bounded, for their own
// copies and MMAs in flight) before TMEM is released.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace fp8q {

using namespace sm100;

namespace {

constexpr int kBM = 128, kBN = 256, kBKB = 128;  // tile rows, tile columns, K bytes per stage
constexpr int kStages = 4;
constexpr int kSbStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kThreads = 320;
constexpr int kGroupM = 16;     // tile rasterization: 16 row tiles share each column sweep
constexpr int kMaxGroups = 256;
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint32_t kAStage = kBM * kBKB;  // 16 KB
constexpr uint32_t kBStage = kBN * kBKB;  // 32 KB

enum { kBlockwise = 0, kMx = 1, kPerTensor = 2, kNvfp4 = 3 };
enum { kFprop = 0, kDgrad = 1, kWgrad = 2 };

template <int R> struct Cfg;
template <> struct Cfg<kBlockwise> { static constexpr uint32_t sfa = 0, sfb = 0, tmem_cols = 512, sf_cols = 0; };
template <> struct Cfg<kPerTensor> { static constexpr uint32_t sfa = 0, sfb = 0, tmem_cols = 256, sf_cols = 0; };
template <> struct Cfg<kMx> { static constexpr uint32_t sfa = 512, sfb = 1024, tmem_cols = 512, sf_cols = 16; };
template <> struct Cfg<kNvfp4> { static constexpr uint32_t sfa = 2048, sfb = 4096, tmem_cols = 512, sf_cols = 64; };

template <int R, int L>
struct Smem {
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + kStages * kAStage;
  static constexpr uint32_t sf = b + kStages * kBStage;
  static constexpr uint32_t sf_stage = Cfg<R>::sfa + Cfg<R>::sfb;
  static constexpr uint32_t sbw = sf + kStages * sf_stage;
  static constexpr uint32_t sbw_bytes = (R == kBlockwise && L == kWgrad) ? kSbStages * kBN * 4 : 0;
  static constexpr uint32_t bars = sbw + sbw_bytes;
  static constexpr uint32_t n_bars = 2 * kStages + 4 + 2 + 2 * kSbStages + 1;
  static constexpr uint32_t misc = bars + n_bars * 8;
  static constexpr uint32_t groups = misc + 16;
  static constexpr uint32_t total = groups + 2 * (kMaxGroups + 1) * 4;
  static constexpr uint32_t alloc = total + 1024;  // room to align the base to 1024 bytes
};

struct Tile {
  int m0, mend, n0, g;
};

// Tile t of the rasterized order: groups of kGroupM row tiles, column-major inside a group.
__device__ __forceinline__ Tile tile_of(int t, const GemmParams& p, int row_tiles, const int* prefix,
                                        const int* offs) {
  const int per = kGroupM * p.tiles_n;
  const int grp = t / per, first = grp * kGroupM;
  const int gsz = min(row_tiles - first, kGroupM);
  const int local = t - grp * per;
  const int rt = first + local % gsz, nt = local / gsz;
  Tile T;
  T.n0 = nt * kBN;
  if (p.num_groups > 0) {
    int g = 0;
    while (g + 1 < p.num_groups && prefix[g + 1] <= rt) ++g;
    T.g = g;
    T.m0 = offs[g] + (rt - prefix[g]) * kBM;
    T.mend = min(offs[g + 1], T.m0 + kBM);
  } else {
    T.g = 0;
    T.m0 = rt * kBM;
    T.mend = min(p.M, T.m0 + kBM);
  }
  return T;
}

__device__ __forceinline__ void raise_timeout(const GemmParams& p, volatile int* abort_flag) {
  *abort_flag = 1;
  atomicExch(p.status, kDevTimeout);
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Stores 8 consecutive results of row m starting at column n (masking the N tail).
__device__ __forceinline__ void store8(const GemmParams& p, int m, int n, const float* v) {
  uint16_t* dst = p.c + (int64_t)m * p.ldc + n;
  if (n + 8 <= p.N) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                                                pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
  } else {
    for (int i = 0; i < 8 && n + i < p.N; ++i) {
      __nv_bfloat16 h = __float2bfloat16_rn(v[i]);
      dst[i] = *reinterpret_cast<uint16_t*>(&h);
    }
  }
}

}  // namespace

template <int R, int L, bool GROUPED>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tma_a,
                const __grid_constant__ CUtensorMap tma_b, const __grid_constant__ CUtensorMap tma_sb) {
  using S = Smem<R, L>;
  constexpr bool kPromote = (R == kBlockwise);
  constexpr bool kWg = kPromote && (L == kWgrad);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::bars);
  uint64_t* empty = full + kStages;
  uint64_t* pfull = empty + kStages;     // [2] partial (or accumulator) ready
  uint64_t* pempty = pfull + 2;          // [2] partial (or accumulator) drained
  uint64_t* final_bar = pempty + 2;      // [2] MMA wind-down
  uint64_t* sbfull = final_bar + 2;
  uint64_t* sbempty = sbfull + kSbStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::misc + 4);
  int* prefix = reinterpret_cast<int*>(smem + S::groups);
  int* offs = prefix + kMaxGroups + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.K / (R == kNvfp4 ? 2 * kBKB : kBKB);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&pfull[i], 1);
      mbar_init(&pempty[i], kEpiWarps * 32);
      mbar_init(&final_bar[i], 1);
    }
    for (int i = 0; i < kSbStages; ++i) {
      mbar_init(&sbfull[i], 1);
      mbar_init(&sbempty[i], kEpiWarps * 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (GROUPED && warp == kProducerWarp) {
    for (int g = lane; g <= p.num_groups; g += 32) offs[g] = p.m_offsets[g];
    __syncwarp();
    if (lane == 0) {
      int acc = 0;
      for (int g = 0; g < p.num_groups; ++g) {
        prefix[g] = acc;
        acc += (offs[g + 1] - offs[g] + kBM - 1) / kBM;
      }
      prefix[p.num_groups] = acc;
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, Cfg<R>::tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int row_tiles = GROUPED ? prefix[p.num_groups] : p.tiles_m;
  const int total = row_tiles * p.tiles_n;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tma_a);
      tma_prefetch_desc(&tma_b);
      if (kWg) tma_prefetch_desc(&tma_sb);
      uint32_t it = 0, sbit = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile T = tile_of(t, p, row_tiles, prefix, offs);
        const int b_row = T.g * p.N + T.n0;
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
          uint32_t tx = kAStage + kBStage;
          if (R == kMx || R == kNvfp4) tx += Cfg<R>::sfa + Cfg<R>::sfb;
          mbar_arrive_expect_tx(&full[s], tx);
          tma_load_2d(smem + S::a + s * kAStage, &tma_a, &full[s], kb * kBKB, T.m0);
          tma_load_2d(smem + S::b + s * kBStage, &tma_b, &full[s], kb * kBKB, b_row);
          if (R == kMx || R == kNvfp4) {
            // scale atoms: 512 bytes per 128 rows x 4 scale columns; MX: 1 atom per chunk,
            // NVFP4: 4 atoms per chunk, for A's row band and B's two row bands.  Bands past
            // the padded buffer end are replaced by A's band (their columns are never stored).
            constexpr uint32_t apc = Cfg<R>::sfa / 512;
            uint8_t* dst = smem + S::sf + s * S::sf_stage;
            const int band_a = T.m0 / kBM;
            bulk_load(dst, p.sfa + ((int64_t)band_a * p.sfa_s4 + (int64_t)kb * apc) * 512, Cfg<R>::sfa, &full[s]);
            const int bands_b = (p.N + kBM - 1) / kBM;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int band = T.n0 / kBM + h;
              const uint8_t* src = (band < bands_b) ? p.sfb + ((int64_t)band * p.sfb_s4 + (int64_t)kb * apc) * 512
                                                    : p.sfb + ((int64_t)kb * apc) * 512;
              bulk_load(dst + Cfg<R>::sfa + h * Cfg<R>::sfa, src, Cfg<R>::sfa, &full[s]);
            }
          }
          if (kWg) {
            const uint32_t ss = sbit % kSbStages, sph = (sbit / kSbStages) & 1;
            if (!mbar_wait(&sbempty[ss], sph ^ 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
            mbar_arrive_expect_tx(&sbfull[ss], kBN * 4);
            tma_load_2d(smem + S::sbw + ss * kBN * 4, &tma_sb, &sbfull[ss], T.n0, kb);
            ++sbit;
          }
        }
      }
      // wind down: every issued stage's copies must land before the CTA exits
      const uint32_t inflight = it < (uint32_t)kStages ? it : (uint32_t)kStages;
      for (uint32_t j = 0; j < inflight; ++j) {
        const uint32_t i2 = it - 1 - j;
        mbar_wait_drain(&full[i2 % kStages], (i2 / kStages) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_dense = (1u << 4) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      constexpr uint32_t idesc_mx = ((uint32_t)(kBN >> 3) << 17) | (1u << 23) | ((uint32_t)(kBM >> 4) << 24);
      constexpr uint32_t idesc_nv = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      uint32_t it = 0, chunk = 0, tiles_done = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tiles_done) {
        if (!kPromote) {
          if (!mbar_wait(&pempty[0], (tiles_done & 1) ^ 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); break; }
          tc_fence_after();
        }
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
          tc_fence_after();
          const uint32_t pb = chunk & 1;
          if (kPromote) {
            if (!mbar_wait(&pempty[pb], ((chunk >> 1) & 1) ^ 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
            tc_fence_after();
          }
          const uint64_t adesc = smem_desc(smem_u32(smem + S::a + s * kAStage), 16, 1024, 2);
          const uint64_t bdesc = smem_desc(smem_u32(smem + S::b + s * kBStage), 16, 1024, 2);
          const uint32_t d = tmem + (kPromote ? pb * kBN : 0);
          if constexpr (R == kBlockwise || R == kPerTensor) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_f8f6f4(d, adesc + 2 * k, bdesc + 2 * k, idesc_dense, (kPromote ? k > 0 : (kb > 0 || k > 0)));
          } else {
            const uint32_t sf_col = kBN + s * Cfg<R>::sf_cols;  // this stage's scale columns
            const uint32_t sfa_t = tmem + sf_col;
            const uint32_t sfb_t = tmem + sf_col + Cfg<R>::sfa / 128;
            const uint32_t sfsm = smem_u32(smem + S::sf + s * S::sf_stage);
            constexpr uint32_t atoms_a = Cfg<R>::sfa / 512;
#pragma unroll
            for (uint32_t a = 0; a < atoms_a; ++a) {
              // A atom a -> 4 columns; B band h atom a -> 4 columns after A's
              tmem_cp_32x128b_x4(sfa_t + 4 * a, smem_desc(sfsm + 512 * a, 0, 128, 0));
#pragma unroll
              for (uint32_t h = 0; h < 2; ++h)
                tmem_cp_32x128b_x4(sfb_t + 8 * a + 4 * h,
                                   smem_desc(sfsm + Cfg<R>::sfa + h * Cfg<R>::sfa + 512 * a, 0, 128, 0));
            }
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
              const uint32_t acc = (kb > 0 || k > 0);
              if constexpr (R == kMx) {
                // MMA k of the chunk uses byte k of each scale column (scale factor id k)
                mma_mxf8(d, adesc + 2 * k, bdesc + 2 * k, idesc_mx | (k << 4) | (k << 29),
                         sfa_t | (k << 30), sfb_t | (k << 30), acc);
              } else {
                // MMA k (64 FP4 values of K) uses the k-th group of 4 (A) / 8 (B) columns
                mma_nvf4(d, adesc + 2 * k, bdesc + 2 * k, idesc_nv, sfa_t + 4 * k, sfb_t + 8 * k, acc);
              }
            }
          }
          mma_commit(&empty[s]);
          if (kPromote) {
            mma_commit(&pfull[pb]);
            ++chunk;
          }
        }
        if (!ok) break;
        if (!kPromote) mma_commit(&pfull[0]);
      }
      // wind down: all MMAs this thread issued complete before TMEM is released
      mma_commit(&final_bar[0]);
      mbar_wait_drain(&final_bar[0], 0, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------------ epilogue warps 0-7
    const int q = warp & 3, wg = warp >> 2;
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(wg * 128);
    const int rloc = q * 32 + lane;
    uint32_t chunk = 0, sbit = 0, tiles_done = 0;
    float alpha = 1.0f;
    if (R == kPerTensor || R == kNvfp4) alpha = __fmul_rn(*p.a_global, *p.b_global);
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tiles_done) {
      const Tile T = tile_of(t, p, row_tiles, prefix, offs);
      const int m = T.m0 + rloc;
      const bool row_ok = m < T.mend;
      const int ncol0 = T.n0 + wg * 128;
      if (kPromote) {
        float2 acc[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) acc[i] = make_float2(0.0f, 0.0f);
        const float* sa_row = p.sa + (m < p.M ? m : 0);
        const bool sa_ok = m < p.M;
        const int nblk = ncol0 / kBM;
        const bool nb_ok = ncol0 < p.N;
        const float* sbg = p.sb + (GROUPED ? (int64_t)T.g * ((p.N + kBM - 1) / kBM) * p.ld_sb : 0);
        float sa_next = sa_ok ? __ldg(sa_row) : 0.0f;
        for (int kb = 0; kb < KB; ++kb) {
          const float sa = sa_next;
          if (kb + 1 < KB) sa_next = sa_ok ? __ldg(sa_row + (int64_t)(kb + 1) * p.ld_sa) : 0.0f;
          float scale = sa;
          if (L == kFprop) scale = nb_ok ? __fmul_rn(sa, __ldg(sbg + (int64_t)nblk * p.ld_sb + kb)) : 0.0f;
          if (L == kDgrad) scale = nb_ok ? __fmul_rn(sa, __ldg(sbg + (int64_t)kb * p.ld_sb + nblk)) : 0.0f;
          const float* sbw = nullptr;
          uint32_t ss = 0;
          if (kWg) {
            ss = sbit % kSbStages;
            if (!mbar_wait(&sbfull[ss], (sbit / kSbStages) & 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
            sbw = reinterpret_cast<const float*>(smem + S::sbw + ss * kBN * 4) + wg * 128;
          }
          const uint32_t pb = chunk & 1;
          if (!mbar_wait(&pfull[pb], (chunk >> 1) & 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
          tc_fence_after();
          // two 16-column TMEM loads in flight per wait
#pragma unroll
          for (int c = 0; c < 8; c += 2) {
            uint32_t r0[16], r1[16];
            tmem_ld_32x32b_x16(t_lane + pb * kBN + c * 16, r0);
            tmem_ld_32x32b_x16(t_lane + pb * kBN + c * 16 + 16, r1);
            tmem_ld_wait(r0);
            tmem_ld_wait(r1);
            if (kWg) {
              const float2 s2 = make_float2(sa, sa);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const float2 b0 = *reinterpret_cast<const float2*>(sbw + c * 16 + 2 * i);
                const float2 b1 = *reinterpret_cast<const float2*>(sbw + c * 16 + 16 + 2 * i);
                const float2 p0 = __fmul2_rn(make_float2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1])), b0);
                const float2 p1 = __fmul2_rn(make_float2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1])), b1);
                acc[c * 8 + i] = __ffma2_rn(p0, s2, acc[c * 8 + i]);
                acc[c * 8 + 8 + i] = __ffma2_rn(p1, s2, acc[c * 8 + 8 + i]);
              }
            } else {
              const float2 s2 = make_float2(scale, scale);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                acc[c * 8 + i] = __ffma2_rn(make_float2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1])), s2,
                                            acc[c * 8 + i]);
                acc[c * 8 + 8 + i] = __ffma2_rn(make_float2(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1])),
                                                s2, acc[c * 8 + 8 + i]);
              }
            }
          }
          tc_fence_before();
          mbar_arrive(&pempty[pb]);
          if (kWg) {
            mbar_arrive(&sbempty[ss]);
            ++sbit;
          }
          ++chunk;
        }
        if (!ok) break;
        if (row_ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = ncol0 + 8 * j;
            if (n < p.N) {
              const float v[8] = {acc[4 * j].x,     acc[4 * j].y,     acc[4 * j + 1].x, acc[4 * j + 1].y,
                                  acc[4 * j + 2].x, acc[4 * j + 2].y, acc[4 * j + 3].x, acc[4 * j + 3].y};
              store8(p, m, n, v);
            }
          }
        }
      } else {
        if (!mbar_wait(&pfull[0], tiles_done & 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); break; }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(t_lane + c * 32, r);
          tmem_ld_wait(r);
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int n = ncol0 + c * 32 + 8 * j;
              if (n < p.N) {
                float v[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(__uint_as_float(r[8 * j + i]), alpha);
                store8(p, m, n, v);
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&pempty[0]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg<R>::tmem_cols);
  }
}

template <int R, int L, bool G>
static cudaError_t launch_one(const GemmParams& p, const CUtensorMap& a, const CUtensorMap& b,
                              const CUtensorMap& sb, int num_sms, cudaStream_t s) {
  auto kern = gemm_kernel<R, L, G>;
  const int smem = (int)Smem<R, L>::alloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int64_t tiles = (int64_t)p.tiles_m * p.tiles_n;
  int grid = (int)(tiles < num_sms ? tiles : num_sms);
  if (grid < 1) grid = 1;
  kern<<<grid, kThreads, smem, s>>>(p, a, b, sb);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmParams& p, const CUtensorMap& tma_a, const CUtensorMap& tma_b,
                        const CUtensorMap& tma_sb, int num_sms, cudaStream_t s) {
  if (p.recipe == kBlockwise) {
    if (p.num_groups > 0) return launch_one<kBlockwise, kFprop, true>(p, tma_a, tma_b, tma_sb, num_sms, s);
    if (p.layout == kFprop) return launch_one<kBlockwise, kFprop, false>(p, tma_a, tma_b, tma_sb, num_sms, s);
    if (p.layout == kDgrad) return launch_one<kBlockwise, kDgrad, false>(p, tma_a, tma_b, tma_sb, num_sms, s);
    return launch_one<kBlockwise, kWgrad, false>(p, tma_a, tma_b, tma_sb, num_sms, s);
  }
  if (p.recipe == kMx) return launch_one<kMx, kFprop, false>(p, tma_a, tma_b, tma_sb, num_sms, s);
  if (p.recipe == kPerTensor) return launch_one<kPerTensor, kFprop, false>(p, tma_a, tma_b, tma_sb, num_sms, s);
  return launch_one<kNvfp4, kFprop, false>(p, tma_a, tma_b, tma_sb, num_sms, s);
}

}  // namespace fp8q
