// Block-scaled low-precision GEMM on the sm_100a tensor cores:
//   C[M x N] (BF16) = A[M x K] . B[N x K]^T with both operands K-major codes.
//
// "Can you explain the role of FP8 precision in DeepSeek-V3 training":
//   "Mixed-precision framework" - the compute-heavy GEMMs run in FP8 (fprop, dgrad, wgrad);
//   "Fine-grained quantization" - 1x128 activation tiles and 128x128 weight blocks;
//   "Increased accumulation precision" - partial results are promoted to FP32 at fixed
//   intervals.  Here the interval is one 128-element K chunk: the tensor cores form the
//   chunk's E4M3 partial product in a TMEM buffer, and CUDA cores add it, times the chunk's
//   two scales, into an FP32 accumulator held in registers (gemm_blockwise_kernel).
// "Accelerating FP8 training performance with the NVIDIA NeMo framework": MXFP8 (block
//   processing in the Blackwell tensor cores: E8M0 scales applied by the MMA itself) and the
//   per-tensor recipe (gemm_scaled_kernel).
// "NVIDIA developed a method to train neural networks in 4-bit precision": NVFP4 (E2M1 with
//   per-16 E4M3 scales applied by the MMA, per-tensor FP32 scales in the epilogue).
//
// Both kernels are persistent (one CTA per SM) and warp-specialized: one warp drives TMA
// into a ring of 128B-swizzled K chunks (128 bytes of K per stage), one warp allocates TMEM
// and a single thread issues tcgen05.mma, the remaining warps drain TMEM (and, for MX and
// NVFP4, four warps store each stage's scale factors into TMEM).
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

constexpr int kBM = 128, kBKB = 128;  // tile rows, K bytes per stage
constexpr int kGroupM = 16;           // rasterization of grouped (expert) GEMMs
constexpr int kMaxGroups = 256;
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr uint32_t kAStage = kBM * kBKB;  // 16 KB

enum { kBlockwise = 0, kMx = 1, kPerTensor = 2, kNvfp4 = 3 };
enum { kFprop = 0, kDgrad = 1, kWgrad = 2 };

struct Tile {
  int m0, mend, n0, g;
};

// Position (row tile, column tile) of tile t in the rasterized order.  Row-grouped
// (p.group_n == 0): groups of p.group_m row tiles, column-major inside a group, so the
// group's A rows stay in L2 while B streams.  Column-grouped (p.group_n > 0): groups of
// p.group_n column tiles, row-major inside a group, so the group's B rows stay in L2 while
// A streams.
__device__ __forceinline__ void raster_pos(int t, const GemmParams& p, int row_tiles, int& rt, int& nt) {
  if (p.group_n > 0) {
    const int per = p.group_n * row_tiles;
    const int grp = t / per, first = grp * p.group_n;
    const int gsz = min(p.tiles_n - first, p.group_n);
    const int local = t - grp * per;
    nt = first + local % gsz;
    rt = local / gsz;
  } else {
    const int per = p.group_m * p.tiles_n;
    const int grp = t / per, first = grp * p.group_m;
    const int gsz = min(row_tiles - first, p.group_m);
    const int local = t - grp * per;
    rt = first + local % gsz;
    nt = local / gsz;
  }
}

// Tile t of the rasterized order for output tiles `bn` columns wide.  Grouped GEMMs
// enumerate each expert's row tiles.
__device__ __forceinline__ Tile tile_of(int t, const GemmParams& p, int row_tiles, const int* prefix,
                                        const int* offs, int bn) {
  int rt, nt;
  raster_pos(t, p, row_tiles, rt, nt);
  Tile T;
  T.n0 = nt * bn;
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

// Blockwise epilogue modes: BF16 C; FP32 C += result; BF16 C plus its 1x128 E4M3 codes.
enum { kEpiBf16 = 0, kEpiAcc32 = 1, kEpiQuant = 2 };

// The two values rounded to BF16 (round to nearest even, as pack_bf16 stores them), as FP32.
__device__ __forceinline__ float2 bf16x2_round(float2 v) {
  return __bfloat1622float2(__floats2bfloat162_rn(v.x, v.y));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Stores 8 consecutive results of row m starting at column n (masking the N tail).
// Eight packed BF16 values at (m, n..n+7); scalar stores past column N.
__device__ __forceinline__ void store8_bf16(const GemmParams& p, int m, int n, uint4 v) {
  uint16_t* dst = p.c + (int64_t)m * p.ldc + n;
  if (n + 8 <= p.N) {
    *reinterpret_cast<uint4*>(dst) = v;
  } else {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    for (int i = 0; i < 8 && n + i < p.N; ++i) dst[i] = (uint16_t)(w[i >> 1] >> (16 * (i & 1)));
  }
}


// C[m, n..n+3] += four FP32 values (FP32 accumulate mode); scalar past column N.
__device__ __forceinline__ void add4_f32(const GemmParams& p, int m, int n, uint4 v) {
  float* dst = p.c32 + (int64_t)m * p.ldc + n;
  const float x[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w)};
  if (n + 4 <= p.N) {
    float4 o = *reinterpret_cast<float4*>(dst);
    o.x = __fadd_rn(o.x, x[0]);
    o.y = __fadd_rn(o.y, x[1]);
    o.z = __fadd_rn(o.z, x[2]);
    o.w = __fadd_rn(o.w, x[3]);
    *reinterpret_cast<float4*>(dst) = o;
  } else {
    for (int i = 0; i < 4 && n + i < p.N; ++i) dst[i] = __fadd_rn(dst[i], x[i]);
  }
}

// ------------------------------------------------------------------ hardware-scaled kernel
// MXFP8, NVFP4 and per-tensor: 128 x 256 output tiles accumulated across all of K in TMEM
// (256 columns per accumulator).  The scale factors of an MX / NVFP4 stage arrive in shared
// memory with its A/B chunk; four scale warps (one per TMEM lane quadrant) move them into the
// stage's TMEM scale columns with tcgen05.st and signal the MMA issuer, so the tensor pipe
// only runs MMAs (a tcgen05.cp per 512-byte atom, issued by the MMA thread, occupied the
// tensor pipe for about as long as the MMAs of an NVFP4 stage).  Per-tensor has no scale
// columns, so it keeps two accumulators and the epilogue of one tile overlaps the MMAs of
// the next; MX / NVFP4 drain their single accumulator before the next tile.
// The epilogue stages BF16 rows through shared memory (width per recipe, as shared memory
// allows) so global stores are contiguous row segments.
constexpr int kBN = 256;
constexpr int kStages = 4;
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kSfWarp0 = 10;   // scale warps 10-13 (MX, NVFP4)
constexpr uint32_t kBStage = kBN * kBKB;  // 32 KB

template <int R> struct Cfg;
// MX / NVFP4 (single accumulator): 16 warps, 128 registers a thread at launch; the two helper
// warpgroups (warps 8-15: producer, MMA, four scale warps, two idle) drop to 40 and the two
// epilogue warpgroups rise to 216, enough to hold a thread's 128 accumulator values, so the
// epilogue takes the whole accumulator out of TMEM, hands it back to the MMA issuer at once
// and scales, converts and stores while the next tile's MMAs run.
template <> struct Cfg<kPerTensor> {
  static constexpr uint32_t sfa = 0, sfb = 0, tmem_cols = 512, acc_bufs = 2, epi_cols = 64;
  static constexpr int threads = 320;
  static constexpr bool split = false;
};
template <> struct Cfg<kMx> {
  static constexpr uint32_t sfa = 512, sfb = 1024, tmem_cols = 512, sf_cols = 16, acc_bufs = 1, epi_cols = 32;
  static constexpr int threads = 512;
  static constexpr bool split = true;
};
template <> struct Cfg<kNvfp4> {
  static constexpr uint32_t sfa = 2048, sfb = 4096, tmem_cols = 512, sf_cols = 64, acc_bufs = 1, epi_cols = 16;
  static constexpr int threads = 512;
  static constexpr bool split = true;
};
constexpr int kSplitRegsLaunch = 128, kSplitRegsEpi = 216, kSplitRegsHelper = 40;
static_assert(2 * 128 * kSplitRegsEpi + 2 * 128 * kSplitRegsHelper <= 512 * kSplitRegsLaunch,
              "register shares exceed the launch pool");

template <int R>
struct Smem {
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + kStages * kAStage;
  static constexpr uint32_t sf = b + kStages * kBStage;
  static constexpr uint32_t sf_stage = Cfg<R>::sfa + Cfg<R>::sfb;
  static constexpr uint32_t stage_c = 32 * Cfg<R>::epi_cols * 2;   // per epilogue warp
  static constexpr uint32_t cst = sf + kStages * sf_stage;
  static constexpr uint32_t bars = cst + kEpiWarps * stage_c;
  static constexpr uint32_t n_bars = 4 * kStages + 2 * Cfg<R>::acc_bufs + 1;
  static constexpr uint32_t misc = bars + n_bars * 8;
  static constexpr uint32_t alloc = misc + 16 + 1024;  // + room to align the base to 1024 bytes
  static_assert(alloc <= 227 * 1024, "shared memory");
};

// Epilogue store of one warp's 32 rows x EC columns (values already scaled, FP32 in `v`,
// lane = row): BF16 rows into the warp's staging buffer (16-byte chunks XOR-swizzled by row,
// bank-conflict free), then CPR = EC / 8 lanes per row store contiguous 16-byte chunks.
template <int EC>
__device__ __forceinline__ void stage_store_rows(uint4* stg, const float* v, const GemmParams& p, int row0,
                                                 int mend, int n0, int lane) {
  constexpr int CPR = EC / 8, RPI = 32 / CPR, SH = CPR == 8 ? 0 : (CPR == 4 ? 1 : 2);
#pragma unroll
  for (int c = 0; c < CPR; ++c) {
    const float* a = v + 8 * c;
    stg[lane * CPR + (c ^ ((lane >> SH) & (CPR - 1)))] =
        make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]), pack_bf16(a[4], a[5]), pack_bf16(a[6], a[7]));
  }
  __syncwarp();
#pragma unroll
  for (int i = 0; i < CPR; ++i) {
    const int r = i * RPI + lane / CPR, c = lane % CPR;
    const uint4 w = stg[r * CPR + (c ^ ((r >> SH) & (CPR - 1)))];
    const int m = row0 + r, n = n0 + c * 8;
    if (m < mend && n < p.N) store8_bf16(p, m, n, w);
  }
  __syncwarp();
}

}  // namespace

template <int R>
__global__ void __launch_bounds__(Cfg<R>::threads, 1)
    gemm_scaled_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tma_a,
                       const __grid_constant__ CUtensorMap tma_b) {
  using S = Smem<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::bars);
  uint64_t* empty = full + kStages;
  constexpr uint32_t kAcc = Cfg<R>::acc_bufs;
  uint64_t* accfull = empty + kStages;   // [kAcc] the tile's accumulator is complete
  uint64_t* accempty = accfull + kAcc;   // [kAcc] the epilogue has drained it
  uint64_t* final_bar = accempty + kAcc; // MMA wind-down
  uint64_t* sfready = final_bar + 1;     // [kStages] MX / NVFP4: the stage's scales are in TMEM
  uint64_t* sffull = sfready + kStages;  // [kStages] MX / NVFP4: the stage's scale bytes landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::misc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = p.K / (R == kNvfp4 ? 2 * kBKB : kBKB);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (uint32_t b = 0; b < kAcc; ++b) {
      mbar_init(&accfull[b], 1);
      mbar_init(&accempty[b], kEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(final_bar, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sfready[i], 4);   // one arrival per scale warp
      mbar_init(&sffull[i], 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, Cfg<R>::tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int total = p.tiles_m * p.tiles_n;

  if (warp >= kEpiWarps) {
  // helper warpgroups: warps 8-11 and 12-15 (MX / NVFP4) give registers to the epilogue
  if constexpr (Cfg<R>::split) reg_dealloc<kSplitRegsHelper>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tma_a);
      tma_prefetch_desc(&tma_b);
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile T = tile_of(t, p, p.tiles_m, nullptr, nullptr, kBN);
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
          // scale atoms: 512 bytes per 128 rows x 4 scale columns; MX: 1 atom per chunk,
          // NVFP4: 4 atoms per chunk, for A's row band and B's two row bands.  A B band past
          // the padded buffer end is replaced by band 0 (its columns are never stored).
          auto load_scales = [&](uint64_t* bar) {
            constexpr uint32_t apc = Cfg<R>::sfa / 512;
            uint8_t* dst = smem + S::sf + s * S::sf_stage;
            const int band_a = T.m0 / kBM;
            bulk_load(dst, p.sfa + ((int64_t)band_a * p.sfa_s4 + (int64_t)kb * apc) * 512, Cfg<R>::sfa, bar);
            const int bands_b = (p.N + kBM - 1) / kBM;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int band = T.n0 / kBM + h;
              const uint8_t* src = (band < bands_b) ? p.sfb + ((int64_t)band * p.sfb_s4 + (int64_t)kb * apc) * 512
                                                    : p.sfb + ((int64_t)kb * apc) * 512;
              bulk_load(dst + Cfg<R>::sfa + h * Cfg<R>::sfa, src, Cfg<R>::sfa, bar);
            }
          };
          // the scale bytes first, on their own barrier, so the scale warps move them into
          // TMEM while the stage's A/B chunk is still in flight
          if constexpr (R != kPerTensor) {
            mbar_arrive_expect_tx(&sffull[s], Cfg<R>::sfa + Cfg<R>::sfb);
            load_scales(&sffull[s]);
          }
          mbar_arrive_expect_tx(&full[s], kAStage + kBStage);
          tma_load_2d(smem + S::a + s * kAStage, &tma_a, &full[s], kb * kBKB, T.m0);
          tma_load_2d(smem + S::b + s * kBStage, &tma_b, &full[s], kb * kBKB, T.n0);
        }
      }
      // wind down: every issued stage's copies must land before the CTA exits
      const uint32_t inflight = it < (uint32_t)kStages ? it : (uint32_t)kStages;
      for (uint32_t j = 0; j < inflight; ++j) {
        const uint32_t i2 = it - 1 - j;
        mbar_wait_drain(&full[i2 % kStages], (i2 / kStages) & 1, kWaitLimitNs);
        if constexpr (R != kPerTensor) mbar_wait_drain(&sffull[i2 % kStages], (i2 / kStages) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // per-tensor operands may be E5M2: a_format bits 7-9, b_format bits 10-12 (E4M3 0, E5M2 1)
      const uint32_t idesc_dense = (1u << 4) | ((uint32_t)p.a_fmt << 7) | ((uint32_t)p.b_fmt << 10) |
                                   ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      constexpr uint32_t idesc_mx = ((uint32_t)(kBN >> 3) << 17) | (1u << 23) | ((uint32_t)(kBM >> 4) << 24);
      constexpr uint32_t idesc_nv = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
      uint32_t it = 0, tiles_done = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tiles_done) {
        const uint32_t ab = tiles_done % kAcc, acc_t = tmem + ab * (uint32_t)kBN;
        if (!mbar_wait(&accempty[ab], ((tiles_done / kAcc) & 1) ^ 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); break; }
        tc_fence_after();
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
          if constexpr (R != kPerTensor) {
            if (!mbar_wait(&sfready[s], ph, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc(smem_u32(smem + S::a + s * kAStage), 16, 1024, 2);
          const uint64_t bdesc = smem_desc(smem_u32(smem + S::b + s * kBStage), 16, 1024, 2);
          if constexpr (R == kPerTensor) {
#pragma unroll
            for (int k = 0; k < 4; ++k) mma_f8f6f4(acc_t, adesc + 2 * k, bdesc + 2 * k, idesc_dense, kb > 0 || k > 0);
          } else {
            const uint32_t sf_col = kBN + s * Cfg<R>::sf_cols;  // this stage's scale columns
            const uint32_t sfa_t = tmem + sf_col;
            const uint32_t sfb_t = tmem + sf_col + Cfg<R>::sfa / 128;
#pragma unroll
            for (uint32_t k = 0; k < 4; ++k) {
              const uint32_t acc = (kb > 0 || k > 0);
              if constexpr (R == kMx) {
                // MMA k of the chunk uses byte k of each scale column (scale factor id k)
                mma_mxf8(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_mx | (k << 4) | (k << 29),
                         sfa_t | (k << 30), sfb_t | (k << 30), acc);
              } else {
                // MMA k (64 FP4 values of K) uses the k-th group of 4 (A) / 8 (B) columns
                mma_nvf4(tmem, adesc + 2 * k, bdesc + 2 * k, idesc_nv, sfa_t + 4 * k, sfb_t + 8 * k, acc);
              }
            }
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&accfull[ab]);
      }
      // wind down: all MMAs this thread issued complete before TMEM is released
      mma_commit(final_bar);
      mbar_wait_drain(final_bar, 0, kWaitLimitNs);
    }
  } else if (warp < kSfWarp0 + 4) {
    // ------------------------------------------------------------------ scale warps 10-13
    // Warp q = warp % 4 writes TMEM lanes 32q..32q+31.  A stage's scales sit in shared memory
    // as 512-byte atoms (128 rows x 4 scale bytes, row r's 4 bytes at (r%32)*16 + (r/32)*4);
    // the block-scaled MMA reads, for its K step a, 4 columns per atom in which lane l of
    // every quadrant holds the atom's 16 bytes l*16..l*16+15.  Each lane therefore stores
    // the same 16 bytes per atom in all four quadrants: A's atoms in 4 columns each, B's two
    // row bands per atom in 4 columns each, after A's.
    if constexpr (R != kPerTensor) {
      constexpr int apc = (int)(Cfg<R>::sfa / 512);   // atoms per stage (MMAs per chunk for NVFP4)
      const uint32_t t_q = tmem + ((uint32_t)((warp & 3) * 32) << 16);
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          // the stage's scale bytes have landed; the MMAs that read this scale slot four
          // chunks ago completed before the producer refilled the stage
          if (!mbar_wait(&sffull[s], ph, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
          tc_fence_after();
          const uint8_t* sm = smem + S::sf + s * S::sf_stage + lane * 16;
          const uint32_t sf_col = kBN + s * Cfg<R>::sf_cols;
          auto ld16 = [&](uint32_t off, uint32_t* v) {   // 16 bytes of one atom row
            const uint4 x = *reinterpret_cast<const uint4*>(sm + off);
            v[0] = x.x, v[1] = x.y, v[2] = x.z, v[3] = x.w;
          };
          if constexpr (apc == 1) {
            uint32_t va[4], vb[8];
            ld16(0, va);
            ld16(Cfg<R>::sfa, vb);
            ld16(2 * Cfg<R>::sfa, vb + 4);
            tmem_st_32x32b_x4(t_q + sf_col, va);
            tmem_st_32x32b_x8(t_q + sf_col + 4, vb);
          } else {
            // 16 columns per store (the warp has 40 registers): A's four atoms, then B's
            // atoms 0-1 and 2-3 with their two row bands each
            uint32_t v[16];
#pragma unroll
            for (int a = 0; a < 4; ++a) ld16(512 * a, v + 4 * a);
            tmem_st_32x32b_x16(t_q + sf_col, v);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              uint32_t w[16];
#pragma unroll
              for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int h = 0; h < 2; ++h) ld16(Cfg<R>::sfa + h * Cfg<R>::sfa + 512 * (2 * g + a), w + 8 * a + 4 * h);
              tmem_st_32x32b_x16(t_q + sf_col + 16 + 16 * g, w);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfready[s]);
        }
      }
    }
  }  // warps 14-15 (MX / NVFP4) only complete the second helper warpgroup
  } else {
    // ------------------------------------------------------------------ epilogue warps 0-7
    if constexpr (Cfg<R>::split) reg_alloc<kSplitRegsEpi>();
    constexpr int EC = (int)Cfg<R>::epi_cols;
    const int q = warp & 3, wg = warp >> 2;
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(wg * 128);
    uint4* stg = reinterpret_cast<uint4*>(smem + S::cst + warp * S::stage_c);
    uint32_t tiles_done = 0;
    float alpha = 1.0f;
    if (R == kPerTensor || R == kNvfp4) alpha = __fmul_rn(*p.a_global, *p.b_global);
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tiles_done) {
      const Tile T = tile_of(t, p, p.tiles_m, nullptr, nullptr, kBN);
      const uint32_t ab = tiles_done % kAcc;
      const int ncol0 = T.n0 + wg * 128;
      if (!mbar_wait(&accfull[ab], (tiles_done / kAcc) & 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); break; }
      tc_fence_after();
      if constexpr (Cfg<R>::split) {
        // the thread's 128 values out of TMEM at once, the accumulator back to the MMA
        // issuer, then scale, convert and store from registers
        uint32_t r[8][16];
#pragma unroll
        for (int h = 0; h < 8; ++h) tmem_ld_32x32b_x16(t_lane + ab * (uint32_t)kBN + h * 16, r[h]);
#pragma unroll
        for (int h = 0; h < 8; ++h) tmem_ld_wait(r[h]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&accempty[ab]);
#pragma unroll
        for (int c = 0; c < 128 / EC; ++c) {
          float v[EC];
#pragma unroll
          for (int i = 0; i < EC; ++i) v[i] = __fmul_rn(__uint_as_float(r[(c * EC + i) / 16][(c * EC + i) % 16]), alpha);
          stage_store_rows<EC>(stg, v, p, T.m0 + q * 32, T.mend, ncol0 + c * EC, lane);
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < 128 / EC; ++c) {
          float v[EC];
#pragma unroll
          for (int h = 0; h < EC / 16; ++h) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(t_lane + ab * (uint32_t)kBN + c * EC + h * 16, r);
            tmem_ld_wait(r);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[h * 16 + i] = __fmul_rn(__uint_as_float(r[i]), alpha);
          }
          stage_store_rows<EC>(stg, v, p, T.m0 + q * 32, T.mend, ncol0 + c * EC, lane);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&accempty[ab]);
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

// ------------------------------------------------------------------ blockwise (promotion) kernel
// CTA pairs (clusters of 2) share 256 x 256 output tiles with the pair MMA
// (tcgen05.mma.cta_group::2, M = 256).  Each CTA loads its own 128 rows of A and its half
// (128 rows) of B, so an SM moves 32 KB per 128-element K chunk instead of 48 KB, and each
// CTA's TMEM receives its 128 rows of the chunk's partial.  The leader CTA's single MMA thread
// issues for both; the TMA completions of both CTAs are counted on the leader's barrier and
// the MMA commits arrive on both CTAs' barriers (multicast commit, no multicast loads).
// In each CTA warps 0-15 promote (warp w: TMEM lanes 32*(w%4).., columns 64*(w/4)..), warp
// 16 drives the A/B TMA, warp 17 owns TMEM (and, in the leader, issues the MMAs) and warp 18
// stages each chunk's scales in a shared-memory ring.  Every promotion thread keeps its 64
// FP32 accumulators in registers for the whole tile, and wgrad's column scales are read from
// shared memory just before their use.  With 19 warps a thread has 96 registers, so fprop and
// dgrad take the partial out of TMEM 16 columns per load and wait; wgrad adds warp 19 to
// complete the helper warpgroup, which hands registers to the promotion warps (112 each) so
// that the next 16-column load is in flight under the current FMAs.  Two 256-column TMEM
// partial buffers (all 512 columns) alternate per K chunk, so the MMAs of chunk k + 1 run while chunk k is promoted;
// the stage's single commit tells both the producers (stage free) and the promotion warps
// (partial complete) of both CTAs.  The per-chunk hand-off between the MMA issuer and the
// promotion warps costs about the same for any tile width, so the widest tile does the most
// MMA work per hand-off.
namespace {

constexpr int kBwPairM = 2 * kBM;               // 256 output rows per pair tile
constexpr int kBwSb = 10;                       // scale ring: chunks of A/B scales staged ahead
constexpr int kBwGo = 10;                       // MMA go barriers: a multiple of both the stage count
                                                // and the two TMEM partial buffers

// Pair tile shape: 256 x 256 outputs, 16 promotion warps.  wgrad (two FP32 operations per
// element and chunk: the column scale, then the row scale) moves registers from the helper
// warpgroup to the promotion warps so that each keeps a TMEM load in flight under its FMAs;
// fprop and dgrad measured faster without the move (their single FMA per element leaves the
// load latency mostly hidden by the other warps).
template <int L>
struct BwCfg {
  static constexpr int BN = (int)kBlockwiseTileN;       // output columns per pair tile
  static constexpr int HalfBN = BN / 2;                 // B rows loaded by each CTA
  static constexpr int EpiWarps = 4 * (BN / 64);        // 32 rows x 64 columns each
  static constexpr int ProducerWarp = EpiWarps, MmaWarp = EpiWarps + 1, ScaleWarp = EpiWarps + 2;
  static constexpr bool Split = (L == kWgrad);           // register reallocation
  static constexpr int IdleWarp = EpiWarps + 3;          // completes the helper warpgroup
  static constexpr int Threads = (EpiWarps + (Split ? 4 : 3)) * 32;
  // Registers per thread: 96 at launch (640 threads, one CTA per SM); the helper warpgroup
  // gives 64 of each thread's back and the promotion warps take 16 more each.
  static constexpr int RegsLaunch = 96, RegsPromo = 112, RegsHelper = 32;
  static_assert(!Split || EpiWarps * 32 * RegsPromo + 128 * RegsHelper <= Threads * RegsLaunch,
                "register shares exceed the launch pool");
  static_assert(ProducerWarp % 4 == 0 && IdleWarp == ProducerWarp + 3,
                "the helper warps form one warpgroup");
  static constexpr uint32_t BStage = HalfBN * kBKB;    // 16 KB
};


// Shared memory of the blockwise kernel.  A scale-ring slot holds one chunk's scales:
// wgrad: [B scales of the tile's 256 columns][A scales of the CTA's 128 rows];
// fprop/dgrad: [A scales][the B scales of the tile's four 64-column groups].
template <int L>
struct BwSmem {
  using C = BwCfg<L>;
  static constexpr bool wg = (L == kWgrad);
  static constexpr int stages = 5;
  static constexpr uint32_t slot_sbw = 0;
  static constexpr uint32_t slot_sa = wg ? C::BN * 4 : 0;
  static constexpr uint32_t slot_sb = slot_sa + kBM * 4;
  static constexpr uint32_t slot_bytes = ((slot_sb + (wg ? 0 : (C::BN / 64) * 4) + 127) / 128) * 128;
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + stages * kAStage;
  static constexpr uint32_t ring = b + stages * C::BStage;
  // epilogue staging per promotion warp: 32 rows x epi_cols BF16 (wgrad: half the width)
  static constexpr int epi_cols = 32;
  static constexpr uint32_t stage_c = 32 * epi_cols * 2;
  // staging buffers 1024-byte aligned: the TMA store's 64-byte swizzle follows address bits
  static constexpr uint32_t cst = ((ring + kBwSb * slot_bytes + 1023) / 1024) * 1024;
  static constexpr uint32_t bars = cst + C::EpiWarps * stage_c;
  static constexpr uint32_t n_bars = kBwGo + stages + 2 * kBwSb + 1 + C::EpiWarps / 2;
  static_assert(kBwGo % stages == 0 && kBwGo % 2 == 0, "go slots must cycle with the stages and TMEM buffers");
  static constexpr uint32_t misc = bars + n_bars * 8;
  static constexpr uint32_t groups = misc + 16;
  // fused output quantization: each promotion warp's 32 row amaxes, read by its partner warp
  static constexpr uint32_t xchg = groups + 2 * (kMaxGroups + 1) * 4;
  static constexpr uint32_t total = xchg + C::EpiWarps * 32 * 4;
  static constexpr uint32_t alloc = total + 1024;
  static_assert(alloc <= 227 * 1024, "shared memory");
};

// Pair tile t: 256 rows x BN columns, rasterized like tile_of; grouped GEMMs enumerate each
// expert's 256-row tiles.  Returns this CTA's 128-row half.
template <int BN>
__device__ __forceinline__ Tile pair_tile_of(int t, const GemmParams& p, int row_tiles, const int* prefix,
                                             const int* offs, uint32_t rank) {
  int rt, nt;
  raster_pos(t, p, row_tiles, rt, nt);
  Tile T;
  T.n0 = nt * BN;
  int end;
  if (p.num_groups > 0) {
    int g = 0;
    while (g + 1 < p.num_groups && prefix[g + 1] <= rt) ++g;
    T.g = g;
    T.m0 = offs[g] + (rt - prefix[g]) * kBwPairM;
    end = offs[g + 1];
  } else {
    T.g = 0;
    T.m0 = rt * kBwPairM;
    end = p.M;
  }
  T.m0 += (int)rank * kBM;
  T.mend = min(end, T.m0 + kBM);
  return T;
}

// Expert row offsets into shared memory, clamped to [previous offset, M] so that no tile
// reaches outside C even when the caller's offsets break their rule (the clamp is recorded
// in the status word), and the prefix count of 256-row pair tiles per expert.
__device__ __forceinline__ void load_pair_groups(const GemmParams& p, int* prefix, int* offs, int lane) {
  for (int g = lane; g <= p.num_groups; g += 32) offs[g] = p.m_offsets[g];
  __syncwarp();
  if (lane == 0) {
    int acc = 0, prev = 0;
    bool bad = false;
    for (int g = 0; g <= p.num_groups; ++g) {
      const int v = offs[g], c = min(max(v, prev), p.M);
      bad |= (c != v);
      offs[g] = prev = c;
    }
    if (bad && blockIdx.x == 0) atomicExch(p.status, kDevBadArg);
    for (int g = 0; g < p.num_groups; ++g) {
      prefix[g] = acc;
      acc += (offs[g + 1] - offs[g] + kBwPairM - 1) / kBwPairM;
    }
    prefix[p.num_groups] = acc;
  }
}

// Work unit t of a launch: the raster index of its pair tile and its K chunks [kb0, kb1).
// Units below main_tiles are whole tiles; with a split last wave, unit main_tiles + u is K
// range u % tail_splits of tile main_tiles + u / tail_splits.
template <bool RANGES>
__device__ __forceinline__ int unit_tile(int t, const GemmParams& p) {
  return (RANGES && t >= p.main_tiles) ? p.main_tiles + (t - p.main_tiles) / p.tail_splits : t;
}
template <bool RANGES>
__device__ __forceinline__ void unit_chunks(int t, const GemmParams& p, int KB, int& kb0, int& kb1) {
  kb0 = 0;
  kb1 = KB;
  if (RANGES && t >= p.main_tiles) {
    const int r = (t - p.main_tiles) % p.tail_splits;
    kb0 = r * KB / p.tail_splits;
    kb1 = (r + 1) * KB / p.tail_splits;
  }
}

}  // namespace

template <int L, bool GROUPED, int EPI>
__global__ void __launch_bounds__(BwCfg<L>::Threads, 1)
    gemm_blockwise_kernel(const __grid_constant__ GemmParams p, const __grid_constant__ CUtensorMap tma_a,
                          const __grid_constant__ CUtensorMap tma_b, const __grid_constant__ CUtensorMap tma_sb,
                          const __grid_constant__ CUtensorMap tma_c, const __grid_constant__ CUtensorMap tma_q) {
  using S = BwSmem<L>;
  constexpr bool kWg = (L == kWgrad);
  constexpr bool ACC32 = EPI == kEpiAcc32, QOUT = EPI == kEpiQuant;
  // BF16 output or FP32 accumulation, not grouped: the last wave may be split into K ranges,
  // whose FP32 partial sums go to the workspace (p.ws, through tma_q) instead of C
  constexpr bool RANGES = (EPI == kEpiBf16 || EPI == kEpiAcc32) && !GROUPED;
  using C = BwCfg<L>;
  constexpr int kBwBN = C::BN, kBwHalfBN = C::HalfBN, kBwEpiWarps = C::EpiWarps;
  constexpr int kBwProducerWarp = C::ProducerWarp, kBwMmaWarp = C::MmaWarp;
  constexpr int kBwScaleWarp = C::ScaleWarp;
  constexpr uint32_t kBwBStage = C::BStage;
  constexpr int kStages = S::stages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // go[c % kBwGo] (leader): chunk c may be issued - both CTAs' A/B halves for c have landed
  // and both CTAs' promotion warps have drained chunk c - 2 from its TMEM buffer.  One barrier
  // per chunk keeps the MMA issuer to a single wait per chunk.
  uint64_t* go = reinterpret_cast<uint64_t*>(smem + S::bars);
  uint64_t* empty = go + kBwGo;        // both CTAs: the stage's MMAs are done (partial ready)
  uint64_t* sfull = empty + kStages;     // local scale ring: slot filled
  uint64_t* sempty = sfull + kBwSb;      // local scale ring: slot read by every promotion warp
  uint64_t* final_bar = sempty + kBwSb;
  uint64_t* xbar = final_bar + 1;        // [EpiWarps/2] fused quantization: partner warps' amaxes
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::misc + 4);
  int* prefix = reinterpret_cast<int*>(smem + S::groups);
  int* offs = prefix + kMaxGroups + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int KB = p.K / kBKB;

  if (threadIdx.x == 0) {
    // go: the leader producer's expect-tx arrival + one per promotion warp of both CTAs
    for (int i = 0; i < kBwGo; ++i) mbar_init(&go[i], 1 + 2 * kBwEpiWarps);
    for (int i = 0; i < kStages; ++i) mbar_init(&empty[i], 1);
    for (int i = 0; i < kBwSb; ++i) {
      mbar_init(&sfull[i], 33);  // lane 0's expect-tx arrival + 32 cp.async arrivals
      mbar_init(&sempty[i], kBwEpiWarps);
    }
    mbar_init(final_bar, 1);
    for (int i = 0; i < kBwEpiWarps / 2; ++i) mbar_init(&xbar[i], 2);
    *abort_flag = 0;
    fence_barrier_init();
    // chunks 0 and 1 have no earlier chunk to drain from their TMEM buffers
    mbar_arrive_count(&go[0], 2 * kBwEpiWarps);
    mbar_arrive_count(&go[1], 2 * kBwEpiWarps);
  }
  if (GROUPED && warp == kBwProducerWarp) load_pair_groups(p, prefix, offs, lane);
  if (warp == kBwMmaWarp) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();   // barriers and TMEM of both CTAs exist before either CTA uses them
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row_tiles = GROUPED ? prefix[p.num_groups] : p.tiles_m;
  const int total = GROUPED ? row_tiles * p.tiles_n
                    : RANGES ? p.main_tiles + (p.tiles_m * p.tiles_n - p.main_tiles) * p.tail_splits
                             : p.main_tiles;
  const int cluster = (int)(blockIdx.x >> 1), n_clusters = (int)(gridDim.x >> 1);

  if (warp >= kBwEpiWarps) {
  // wgrad: the helper warpgroup (warps 16-19) gives registers to the promotion warps
  if constexpr (C::Split) reg_dealloc<C::RegsHelper>();
  if (warp == kBwProducerWarp) {
    // ------------------------------------------------------------------ A / B producer
    // One thread: wait for a free stage, arm the leader's barrier, issue the two TMA loads.
    // Nothing else runs on this thread, so it stays several chunks ahead of the MMAs.
    if (lane == 0) {
      tma_prefetch_desc(&tma_a);
      tma_prefetch_desc(&tma_b);
      uint32_t it = 0;
      bool ok = true;
      for (int t = cluster; t < total && ok; t += n_clusters) {
        const Tile T = pair_tile_of<kBwBN>(unit_tile<RANGES>(t, p), p, row_tiles, prefix, offs, rank);
        const int b_row = T.g * p.N + T.n0 + (int)rank * kBwHalfBN;
        int kb0, kb1;
        unit_chunks<RANGES>(t, p, KB, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const uint32_t s = it % kStages, ph = (it / kStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, kWaitLimitNs)) {
            raise_timeout(p, abort_flag);
            ok = false;
            break;
          }
          const uint32_t g = it % kBwGo;
          if (leader) mbar_arrive_expect_tx(&go[g], 2 * (kAStage + kBwBStage));
          const uint32_t bar = mapa_shared(smem_u32(&go[g]), 0);
          tma_load_2d_pair(smem + S::a + s * kAStage, &tma_a, bar, kb * kBKB, T.m0);
          tma_load_2d_pair(smem + S::b + s * kBwBStage, &tma_b, bar, kb * kBKB, b_row);
        }
      }
      if (leader) {  // the leader's go barriers see both halves: wait for the copies in flight
        const uint32_t inflight = it < (uint32_t)kStages ? it : (uint32_t)kStages;
        for (uint32_t j = 0; j < inflight; ++j) {
          const uint32_t i2 = it - 1 - j;
          mbar_wait_drain(&go[i2 % kBwGo], (i2 / kBwGo) & 1, kWaitLimitNs);
        }
      }
    }
  } else if (warp == kBwScaleWarp) {
    // ------------------------------------------------------------------ scale loader
    // All 32 lanes copy each chunk's scales into the scale ring with cp.async (the wgrad
    // B-scale row by TMA); a slot's barrier completes once every lane's copies have landed,
    // so the promotion warps read scales from shared memory only.
    if (kWg && lane == 0) tma_prefetch_desc(&tma_sb);
    uint32_t it = 0;
    bool ok = true;
    for (int t = cluster; t < total && ok; t += n_clusters) {
      const Tile T = pair_tile_of<kBwBN>(unit_tile<RANGES>(t, p), p, row_tiles, prefix, offs, rank);
      const float* sbg = p.sb + (GROUPED ? (int64_t)T.g * ((p.N + kBM - 1) / kBM) * p.ld_sb : 0);
      int kb0, kb1;
      unit_chunks<RANGES>(t, p, KB, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const uint32_t r = it % kBwSb, rph = (it / kBwSb) & 1;
        int good = 1;
        if (lane == 0) {
          good = mbar_wait(&sempty[r], rph ^ 1, abort_flag, kWaitLimitNs);
          if (!good) raise_timeout(p, abort_flag);
        }
        if (!__shfl_sync(0xFFFFFFFFu, good, 0)) { ok = false; break; }
        uint8_t* slot = smem + S::ring + r * S::slot_bytes;
        float* ssa = reinterpret_cast<float*>(slot + S::slot_sa);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int m = T.m0 + i * 32 + lane;
          const bool in = m < p.M;
          cp_async_4(ssa + i * 32 + lane, p.sa + (in ? (int64_t)kb * p.ld_sa + m : 0), in ? 4u : 0u);
        }
        if (!kWg && lane < kBwBN / 64) {
          const int ncol0 = T.n0 + lane * 64, nblk = ncol0 / kBM;
          const bool in = ncol0 < p.N;
          const int64_t off = !in ? 0 : (L == kFprop) ? (int64_t)nblk * p.ld_sb + kb : (int64_t)kb * p.ld_sb + nblk;
          cp_async_4(reinterpret_cast<float*>(slot + S::slot_sb) + lane, sbg + off, in ? 4u : 0u);
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&sfull[r], kWg ? kBwBN * 4 : 0);
          if (kWg) tma_load_2d(slot + S::slot_sbw, &tma_sb, &sfull[r], T.n0, kb);
        }
        cp_async_arrive_noinc(&sfull[r]);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // no scale copy outlives the CTA
    if (kWg && lane == 0) {  // the wgrad B-scale TMA of the last slots
      const uint32_t inflight = it < (uint32_t)kBwSb ? it : (uint32_t)kBwSb;
      for (uint32_t j = 0; j < inflight; ++j) {
        const uint32_t i2 = it - 1 - j;
        mbar_wait_drain(&sfull[i2 % kBwSb], (i2 / kBwSb) & 1, kWaitLimitNs);
      }
    }
  } else if (warp == kBwMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = (1u << 4) | ((uint32_t)(kBwBN >> 3) << 17) | ((uint32_t)(kBwPairM >> 4) << 24);
      uint32_t it = 0;
      bool ok = true;
      for (int t = cluster; t < total && ok; t += n_clusters) {
        int kb0, kb1;
        unit_chunks<RANGES>(t, p, KB, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const uint32_t s = it % kStages, pb = it & 1;
          if (!mbar_wait(&go[it % kBwGo], (it / kBwGo) & 1, abort_flag, kWaitLimitNs)) {
            raise_timeout(p, abort_flag);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = smem_desc(smem_u32(smem + S::a + s * kAStage), 16, 1024, 2);
          const uint64_t bdesc = smem_desc(smem_u32(smem + S::b + s * kBwBStage), 16, 1024, 2);
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_f8f6f4_pair(tmem + pb * kBwBN, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0);
          // one commit per chunk: the stage is free for the producers and the partial is in
          // TMEM for the promotion warps of both CTAs
          mma_commit_pair(&empty[s], 0x3);
        }
      }
      mma_commit_pair(final_bar, 0x1);
      mbar_wait_drain(final_bar, 0, kWaitLimitNs);
    }
  }  // wgrad: warp 19 only completes the helper warpgroup
  } else {
    // ------------------------------------------------------------------ promotion warps 0-15
    // wgrad: 64 accumulators plus two 16-column partials in flight
    if constexpr (C::Split) reg_alloc<C::RegsPromo>();
    const int q = warp & 3, cgp = warp >> 2;
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(cgp * 64);
    const int rloc = q * 32 + lane;
    const uint32_t go_leader = mapa_shared(smem_u32(&go[0]), 0);   // the leader's go[0]
    uint32_t chunk = 0, tile_it = 0;
    bool ok = true;
    for (int t = cluster; t < total && ok; t += n_clusters, ++tile_it) {
      const Tile T = pair_tile_of<kBwBN>(unit_tile<RANGES>(t, p), p, row_tiles, prefix, offs, rank);
      const int ncol0 = T.n0 + cgp * 64;
      float2 acc[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) acc[i] = make_float2(0.0f, 0.0f);
      int kb0, kb1;
      unit_chunks<RANGES>(t, p, KB, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb) {
        const uint32_t rs = chunk % kBwSb;
        if (!mbar_wait(&sfull[rs], (chunk / kBwSb) & 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
        const uint8_t* slot = smem + S::ring + rs * S::slot_bytes;
        const float sa = reinterpret_cast<const float*>(slot + S::slot_sa)[rloc];
        const float sbv = kWg ? 1.0f : reinterpret_cast<const float*>(slot + S::slot_sb)[cgp];
        const float* sbw = reinterpret_cast<const float*>(slot + S::slot_sbw) + cgp * 64;
        const uint32_t pb = chunk & 1;
        // the stage's commit also means: this chunk's partial is complete in TMEM buffer pb
        if (!mbar_wait(&empty[chunk % kStages], (chunk / kStages) & 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
        tc_fence_after();
        const float scale = kWg ? sa : __fmul_rn(sa, sbv);
        const float2 s2 = make_float2(scale, scale);
        // 16-column group h of the partial, times the chunk's scales, into the accumulators
        // (wgrad also scales each column: its B scales are per column and chunk)
        auto fma16 = [&](const uint32_t (&r)[16], int h) {
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            float2 p0 = make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
            float2 p1 = make_float2(__uint_as_float(r[2 * i + 2]), __uint_as_float(r[2 * i + 3]));
            if constexpr (kWg) {
              const float4 c = ld_shared_f4(sbw + h * 16 + 2 * i);
              p0 = __fmul2_rn(p0, make_float2(c.x, c.y));
              p1 = __fmul2_rn(p1, make_float2(c.z, c.w));
            }
            acc[h * 8 + i] = __ffma2_rn(p0, s2, acc[h * 8 + i]);
            acc[h * 8 + i + 1] = __ffma2_rn(p1, s2, acc[h * 8 + i + 1]);
          }
        };
        const uint32_t tb = t_lane + pb * kBwBN;
        const uint32_t go_rel = go_leader + 8u * ((chunk + 2) % kBwGo);  // chunk + 2 reuses pb
        if constexpr (C::Split) {
          // the next group's load is in flight while a group's FMAs run; once the last group
          // is in registers the TMEM buffer goes back to the MMA issuer, before its FMAs
          uint32_t ra[16], rb[16];
          tmem_ld_32x32b_x16(tb, ra);
          tmem_ld_wait(ra);
          tmem_ld_32x32b_x16(tb + 16, rb);
          fma16(ra, 0);
          tmem_ld_wait(rb);
          tmem_ld_32x32b_x16(tb + 32, ra);
          fma16(rb, 1);
          tmem_ld_wait(ra);
          tmem_ld_32x32b_x16(tb + 48, rb);
          fma16(ra, 2);
          tmem_ld_wait(rb);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(go_rel);
          fma16(rb, 3);
        } else {
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(tb + h * 16, r);
            tmem_ld_wait(r);
            fma16(r, h);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(go_rel);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_relaxed(&sempty[rs]);   // the chunk's scales are read
        ++chunk;
      }
      if (!ok) break;
      // Epilogue through this warp's staging buffer: each lane writes its row's values as
      // 16-byte chunks XOR-swizzled by row (conflict-free), then CPR lanes per row move the
      // row's contiguous bytes (128 B per row for fprop/dgrad, 64 B for wgrad), 32 / CPR
      // rows per instruction.  BF16 output: 8 values per chunk, stored.  FP32 accumulate:
      // 4 values per chunk, added to C in FP32.
      constexpr int EC = S::epi_cols, CPR = EC / 8, RPI = 32 / CPR;
      auto swz = [](int r) { return CPR == 8 ? (r & 7) : ((r >> 1) & 3); };
      uint4* stg = reinterpret_cast<uint4*>(smem + S::cst + warp * S::stage_c);
      if (RANGES && t >= p.main_tiles) {
        // a K range of a split tile: its FP32 partial sum goes, in the same 32 x 16 boxes as
        // the FP32-accumulate epilogue, to this unit's own workspace rows by TMA store
        const int wrow = (t - p.main_tiles) * kBwPairM + (int)rank * kBM + q * 32;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          if (lane == 0) bulk_wait_read();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < CPR; ++c) {
            const float2* a2 = acc + h * 8 + c * 2;
            stg[lane * CPR + (c ^ swz(lane))] = make_uint4(__float_as_uint(a2[0].x), __float_as_uint(a2[0].y),
                                                           __float_as_uint(a2[1].x), __float_as_uint(a2[1].y));
          }
          fence_proxy_async();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tma_q, stg, cgp * 64 + h * 16, wrow);
            bulk_commit();
          }
        }
        continue;
      }
      if constexpr (!ACC32) {
        // BF16: the staged 32 x 32 box goes out by one TMA store and the warp moves on to the
        // next tile while the copy engine writes it (the swizzled staging layout is the tensor
        // map's 64-byte swizzle); the box is reused only after the store has read it.  A
        // grouped GEMM's box that would reach past its expert's rows is stored by the warp.
        const bool tma_box = !GROUPED || T.m0 + q * 32 + 32 <= T.mend;
#pragma unroll
        for (int h = 0; h < 64 / EC; ++h) {
          if (lane == 0) bulk_wait_read();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < CPR; ++c) {
            const float2* a4 = acc + h * (EC / 2) + c * 4;
            stg[lane * CPR + (c ^ swz(lane))] = make_uint4(pack_bf16(a4[0].x, a4[0].y), pack_bf16(a4[1].x, a4[1].y),
                                                           pack_bf16(a4[2].x, a4[2].y), pack_bf16(a4[3].x, a4[3].y));
          }
          if (tma_box) {
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&tma_c, stg, ncol0 + h * EC, T.m0 + q * 32);
              bulk_commit();
            }
            continue;
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < CPR; ++i) {
            const int r = i * RPI + lane / CPR, c = lane % CPR;
            const uint4 v = stg[r * CPR + (c ^ swz(r))];
            const int mr = T.m0 + q * 32 + r, n = ncol0 + h * EC + c * 8;
            if (mr < T.mend && n < p.N) store8_bf16(p, mr, n, v);
          }
          __syncwarp();
        }
      } else {
        constexpr int EC32 = EC / 2;   // FP32 columns per pass (same bytes per row)
        // the staged 32 x 16 FP32 box is added into C by one TMA reduction (C + S rounded to
        // FP32 once per element, as below); a grouped box reaching past its expert's rows is
        // added by the warp
        const bool tma_box = !GROUPED || T.m0 + q * 32 + 32 <= T.mend;
#pragma unroll
        for (int h = 0; h < 64 / EC32; ++h) {
          if (lane == 0) bulk_wait_read();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < CPR; ++c) {
            const float2* a2 = acc + h * (EC32 / 2) + c * 2;
            stg[lane * CPR + (c ^ swz(lane))] = make_uint4(__float_as_uint(a2[0].x), __float_as_uint(a2[0].y),
                                                           __float_as_uint(a2[1].x), __float_as_uint(a2[1].y));
          }
          if (tma_box) {
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_2d(&tma_c, stg, ncol0 + h * EC32, T.m0 + q * 32);
              bulk_commit();
            }
            continue;
          }
          __syncwarp();
#pragma unroll
          for (int i = 0; i < CPR; ++i) {
            const int r = i * RPI + lane / CPR, c = lane % CPR;
            const uint4 v = stg[r * CPR + (c ^ swz(r))];
            const int mr = T.m0 + q * 32 + r, n = ncol0 + h * EC32 + c * 4;
            if (mr < T.mend && n < p.N) add4_f32(p, mr, n, v);
          }
          __syncwarp();
        }
      }
      if constexpr (QOUT) {
        // Fused 1x128 quantization of the BF16 output along N (the next layer's activation
        // codes and scales, as the 1x128 rowwise quantizer would make them from C): a
        // 128-column group of a row is this warp's 64 columns and those of warp ^ 4, so the
        // two warps' row amaxes meet in shared memory behind a two-arrival barrier.
        float am = 0.0f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {     // the values just stored, rounded to BF16
          acc[j] = bf16x2_round(acc[j]);
          am = fmaxf(am, fmaxf(fabsf(acc[j].x), fabsf(acc[j].y)));
        }
        float* xch = reinterpret_cast<float*>(smem + S::xchg);
        xch[warp * 32 + lane] = am;
        __syncwarp();
        uint64_t* xb = &xbar[q * 2 + (cgp >> 1)];
        if (lane == 0) mbar_arrive(xb);   // release: the warp's amaxes are visible
        if (!mbar_wait(xb, tile_it & 1, abort_flag, kWaitLimitNs)) { raise_timeout(p, abort_flag); ok = false; break; }
        am = fmaxf(am, xch[(warp ^ 4) * 32 + lane]);
        const float sf = e4m3_sf(am);
        const float2 s2 = make_float2(sf, sf);
        if (lane == 0) bulk_wait_read();     // the BF16 box store has read the buffer
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 4; ++c) {        // 16 codes (16 bytes) per chunk of the lane's row
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 y0 = __fmul2_rn(acc[c * 8 + 2 * k], s2);
            const float2 y1 = __fmul2_rn(acc[c * 8 + 2 * k + 1], s2);
            w[k] = cvt_e4m3x2(y0.x, y0.y) | (cvt_e4m3x2(y1.x, y1.y) << 16);
          }
          stg[lane * 4 + (c ^ swz(lane))] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        // the 32 x 64 code box (same 64-byte swizzle) goes out by TMA store as well
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&tma_q, stg, ncol0, T.m0 + q * 32);
          bulk_commit();
        }
        const int mrow = T.m0 + q * 32 + lane;
        if ((cgp & 1) == 0 && mrow < T.mend && ncol0 < p.N)
          p.s_out[(int64_t)(ncol0 >> 7) * p.ld_s_out + mrow] = __frcp_rn(sf);
      }
    }
  }

  if (warp < kBwEpiWarps && lane == 0) bulk_wait_all();   // the epilogue's TMA stores are done
  tc_fence_before();
  __syncwarp();     // role loops ran on lane 0 only: reconverge before the aligned barrier
  cluster_sync();   // the leader's MMAs into both TMEMs are complete before either frees
  if (warp == kBwMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Raster (which operand stays in L2).  Concurrent tiles should share operands in L2 and the
// operand that is re-read across sweeps should stay resident.  When A is the smaller operand
// (M <= N) groups of row tiles (about 40 MB of A) sweep all column tiles: A stays resident,
// B streams through once per group.  Otherwise groups of column tiles (about 40 MB of B)
// sweep all row tiles: B stays resident, A streams through once per group.  Grouped (expert)
// GEMMs keep groups of kGroupM row tiles.
static void raster(GemmParams& q, int row_tiles, int tile_m, int tile_n) {
  q.group_n = 0;
  if (q.num_groups > 0) {
    q.group_m = kGroupM;
    return;
  }
  const int64_t kbytes = q.recipe == kNvfp4 ? q.K / 2 : q.K;
  if (q.M <= q.N) {
    int64_t g = (40ll << 20) / max((int64_t)tile_m * kbytes, (int64_t)1);
    q.group_m = (int)max((int64_t)1, min(g, (int64_t)row_tiles));
  } else {
    q.group_m = 1;
    int64_t g = (40ll << 20) / max((int64_t)tile_n * kbytes, (int64_t)1);
    q.group_n = (int)max((int64_t)1, min(g, (int64_t)q.tiles_n));
  }
}

// Launch configuration of one blockwise instantiation: its shared memory, the register check
// of the register-moving (wgrad) form, and how many CTA pairs can be resident at once.
template <int L, bool G, int EPI>
static cudaError_t blockwise_config(cudaLaunchConfig_t& cfg, cudaLaunchAttribute* attr, int num_sms, cudaStream_t s,
                                    int& pairs) {
  auto kern = gemm_blockwise_kernel<L, G, EPI>;
  using C = BwCfg<L>;
  // The register reallocation inside the wgrad kernel adds up to exactly the launch pool at
  // 96 registers per thread; with any other count an increase could wait forever, so refuse.
  if constexpr (C::Split) {
    static const int regs = [] {
      cudaFuncAttributes fa{};
      return cudaFuncGetAttributes(&fa, gemm_blockwise_kernel<L, G, EPI>) == cudaSuccess ? fa.numRegs : -1;
    }();
    if (regs != C::RegsLaunch) return cudaErrorInvalidConfiguration;
  }
  const int smem = (int)BwSmem<L>::alloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cfg = cudaLaunchConfig_t{};
  cfg.gridDim = dim3(num_sms - (num_sms & 1));
  cfg.blockDim = dim3(C::Threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int resident = 0;
  e = cudaOccupancyMaxActiveClusters(&resident, kern, &cfg);
  if (e != cudaSuccess) return e;
  pairs = resident < num_sms / 2 ? resident : num_sms / 2;
  if (pairs < 1) pairs = 1;
  return cudaSuccess;
}

// Output tiles of a blockwise GEMM (256-row pair tiles x 256 columns) with its raster.
static void blockwise_grid(GemmParams& q, bool grouped) {
  q.tiles_n = (q.N + kBlockwiseTileN - 1) / kBlockwiseTileN;
  q.tiles_m = (q.M + kBwPairM - 1) / kBwPairM + (grouped ? q.num_groups : 0);
  raster(q, q.tiles_m, kBwPairM, kBlockwiseTileN);
}

// Split of the last, partial wave: with `pairs` persistent CTA pairs, `tiles` tiles leave
// tiles % pairs for a last wave in which most pairs are idle for a whole tile.  When that
// wave is at most half full, its tiles are cut into `splits` K ranges of at least 4 chunks
// (at most one range per pair), run after the whole tiles in the same launch, so the wave
// takes about 1 / splits of a tile's time; the ranges' FP32 partial sums go to a workspace
// and a small kernel adds them and rounds to BF16.  The ranges' FP32 stores, the sum kernel
// and its launch cost about as much as 10-15 chunks of a tile (Llama-3-8B on 256 x 256
// tiles: wgrad, 64 chunks cut 9 ways, -4.9%; fprop, 32 chunks cut 4 ways, -0.8%), so the
// split is taken only when it saves at least kTailMinSaved chunks of the last wave.
// Returns the workspace bytes (0: no split).
constexpr int kTailMinSaved = 16;
static int64_t tail_plan(int64_t tiles, int pairs, int KB, int& tail, int& splits) {
  tail = (int)(tiles % pairs);
  splits = 0;
  if (tail == 0 || 2 * tail > pairs) return 0;
  const int s = min(pairs / tail, KB / 4);
  if (s < 2 || KB - (KB + s - 1) / s < kTailMinSaved) return 0;
  splits = s;
  return (int64_t)tail * s * kBwPairM * kBlockwiseTileN * (int64_t)sizeof(float);
}

// Split tail, last step: each thread adds the K-range partial sums of 8 columns of one row of
// a tail tile in range order (FP32) and stores them as BF16 into C or, when accumulating in
// FP32, adds the sum into C (one addition per element), masked at M and N; a CTA covers 8
// rows, 32 CTAs a tile.
__global__ void __launch_bounds__(256) blockwise_tail_sum_kernel(const __grid_constant__ GemmParams p) {
  const int u = blockIdx.x >> 5, r = (blockIdx.x & 31) * 8 + (threadIdx.x >> 5);
  int rt, nt;
  raster_pos(p.main_tiles + u, p, p.tiles_m, rt, nt);
  const int c = (threadIdx.x & 31) * 8;
  const int m = rt * kBwPairM + r, n = nt * (int)kBlockwiseTileN + c;
  if (m >= p.M || n >= p.N) return;
  constexpr int64_t kRange = (int64_t)kBwPairM * kBlockwiseTileN / 4;   // float4s per K range
  const float4* w = reinterpret_cast<const float4*>(p.ws) + (int64_t)u * p.tail_splits * kRange +
                    ((int64_t)r * kBlockwiseTileN + c) / 4;
  float4 lo = __ldg(w), hi = __ldg(w + 1);
#pragma unroll 4
  for (int k = 1; k < p.tail_splits; ++k) {
    const float4 a = __ldg(w + k * kRange), b = __ldg(w + k * kRange + 1);
    lo = make_float4(__fadd_rn(lo.x, a.x), __fadd_rn(lo.y, a.y), __fadd_rn(lo.z, a.z), __fadd_rn(lo.w, a.w));
    hi = make_float4(__fadd_rn(hi.x, b.x), __fadd_rn(hi.y, b.y), __fadd_rn(hi.z, b.z), __fadd_rn(hi.w, b.w));
  }
  if (p.c32 != nullptr) {
    add4_f32(p, m, n, make_uint4(__float_as_uint(lo.x), __float_as_uint(lo.y), __float_as_uint(lo.z),
                                 __float_as_uint(lo.w)));
    add4_f32(p, m, n + 4, make_uint4(__float_as_uint(hi.x), __float_as_uint(hi.y), __float_as_uint(hi.z),
                                     __float_as_uint(hi.w)));
  } else {
    store8_bf16(p, m, n, make_uint4(pack_bf16(lo.x, lo.y), pack_bf16(lo.z, lo.w), pack_bf16(hi.x, hi.y),
                                    pack_bf16(hi.z, hi.w)));
  }
}

template <int L, bool G, int EPI = kEpiBf16>
static cudaError_t launch_blockwise(const GemmParams& p, const CUtensorMap& a, const CUtensorMap& b,
                                    const CUtensorMap& sb, const CUtensorMap& c, const CUtensorMap& qm,
                                    const CUtensorMap& ws, int num_sms, cudaStream_t s) {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  int pairs = 1;
  cudaError_t e = blockwise_config<L, G, EPI>(cfg, attr, num_sms, s, pairs);
  if (e != cudaSuccess) return e;
  GemmParams q = p;
  blockwise_grid(q, G);
  const int64_t tiles = (int64_t)q.tiles_m * q.tiles_n;
  if (tiles > (int64_t)INT32_MAX / 2) return cudaErrorInvalidValue;
  q.main_tiles = (int)tiles;
  q.tail_splits = 0;
  int tail = 0, splits = 0;
  if constexpr ((EPI == kEpiBf16 || EPI == kEpiAcc32) && !G) {
    // the split ranges run as extra units of this launch, after the whole tiles
    const int64_t need = tail_plan(tiles, pairs, p.K / kBKB, tail, splits);
    if (need > 0 && p.ws != nullptr && p.ws_bytes >= need) {
      q.main_tiles = (int)(tiles - tail);
      q.tail_splits = splits;
    } else {
      splits = 0;
    }
  }
  const int64_t units = q.main_tiles + (int64_t)tail * splits;
  cfg.gridDim = dim3(2 * (int)min((int64_t)pairs, units));
  // tma_q carries the workspace map when the last wave is split (the BF16 and FP32-accumulate
  // epilogues have no fused quantization)
  e = cudaLaunchKernelEx(&cfg, gemm_blockwise_kernel<L, G, EPI>, q, a, b, sb, c, splits > 0 ? ws : qm);
  if (e != cudaSuccess) return e;
  if (splits > 0) {
    blockwise_tail_sum_kernel<<<tail * 32, 256, 0, s>>>(q);
    return cudaGetLastError();
  }
  return cudaSuccess;
}

size_t blockwise_workspace_bytes(const GemmParams& p, int num_sms) {
  if (p.recipe != kBlockwise || p.q_out != nullptr || p.num_groups > 0) return 0;
  if (p.M <= 0 || p.N <= 0 || p.K <= 0) return 0;
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  int pairs = 1;
  cudaError_t e = p.layout == kFprop   ? blockwise_config<kFprop, false, kEpiBf16>(cfg, attr, num_sms, 0, pairs)
                  : p.layout == kDgrad ? blockwise_config<kDgrad, false, kEpiBf16>(cfg, attr, num_sms, 0, pairs)
                                       : blockwise_config<kWgrad, false, kEpiBf16>(cfg, attr, num_sms, 0, pairs);
  if (e != cudaSuccess) return 0;
  GemmParams q = p;
  blockwise_grid(q, false);
  int tail = 0, splits = 0;
  return (size_t)tail_plan((int64_t)q.tiles_m * q.tiles_n, pairs, p.K / kBKB, tail, splits);
}

template <int R>
static cudaError_t launch_scaled(const GemmParams& p, const CUtensorMap& a, const CUtensorMap& b, int num_sms,
                                 cudaStream_t s) {
  auto kern = gemm_scaled_kernel<R>;
  // The register reallocation of MX / NVFP4 adds up to exactly the launch pool at 128
  // registers per thread; with any other count an increase could wait forever, so refuse.
  if constexpr (Cfg<R>::split) {
    static const int regs = [] {
      cudaFuncAttributes fa{};
      return cudaFuncGetAttributes(&fa, gemm_scaled_kernel<R>) == cudaSuccess ? fa.numRegs : -1;
    }();
    if (regs != kSplitRegsLaunch) return cudaErrorInvalidConfiguration;
  }
  const int smem = (int)Smem<R>::alloc;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  GemmParams q = p;
  q.tiles_n = (p.N + kBN - 1) / kBN;
  raster(q, q.tiles_m, kBM, kBN);
  const int64_t tiles = (int64_t)q.tiles_m * q.tiles_n;
  int grid = (int)(tiles < num_sms ? tiles : num_sms);
  if (grid < 1) grid = 1;
  kern<<<grid, Cfg<R>::threads, smem, s>>>(q, a, b);
  return cudaGetLastError();
}

// Failure-detection self test: one thread waits on a barrier nothing arrives on; the bounded
// wait gives up after limit_ns and records the timeout like a GEMM role would.
__global__ void __launch_bounds__(32) selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag, limit_ns)) atomicExch(status, kDevTimeout);
}

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmParams& p, const CUtensorMap& tma_a, const CUtensorMap& tma_b,
                        const CUtensorMap& tma_sb, const CUtensorMap& tma_c, const CUtensorMap& tma_q,
                        const CUtensorMap& tma_ws, int num_sms, cudaStream_t s) {
  if (p.recipe == kBlockwise) {
    if (p.c32 != nullptr) {   // FP32 accumulate epilogue: its own instantiations
      if (p.num_groups > 0) return launch_blockwise<kFprop, true, kEpiAcc32>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
      if (p.layout == kFprop) return launch_blockwise<kFprop, false, kEpiAcc32>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
      if (p.layout == kDgrad) return launch_blockwise<kDgrad, false, kEpiAcc32>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
      return launch_blockwise<kWgrad, false, kEpiAcc32>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
    }
    if (p.q_out != nullptr) {  // BF16 output plus its fused 1x128 quantization
      if (p.layout == kFprop) return launch_blockwise<kFprop, false, kEpiQuant>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
      if (p.layout == kDgrad) return launch_blockwise<kDgrad, false, kEpiQuant>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
      return launch_blockwise<kWgrad, false, kEpiQuant>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
    }
    if (p.num_groups > 0) return launch_blockwise<kFprop, true>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
    if (p.layout == kFprop) return launch_blockwise<kFprop, false>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
    if (p.layout == kDgrad) return launch_blockwise<kDgrad, false>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
    return launch_blockwise<kWgrad, false>(p, tma_a, tma_b, tma_sb, tma_c, tma_q, tma_ws, num_sms, s);
  }
  if (p.recipe == kMx) return launch_scaled<kMx>(p, tma_a, tma_b, num_sms, s);
  if (p.recipe == kPerTensor) return launch_scaled<kPerTensor>(p, tma_a, tma_b, num_sms, s);
  return launch_scaled<kNvfp4>(p, tma_a, tma_b, num_sms, s);
}

}  // namespace fp8q
