// kvq_encode_tc.cu -- the SRFT-int4 encode on the 5th-generation tensor cores.
//
// The encode of "When Quantization Is Free" (gist.science/de/paper/2605.05699,
// "Methodik" 1-2) is linear up to the quantiser: y = Lambda F_r diag(s) x. For a
// tile of 128 vectors this is a GEMM Y[128 x D] = X[128 x D] W^T with the
// per-plan matrix W = Lambda F_r diag(s), which tcgen05.mma runs with fp32
// accumulators in tensor memory (TMEM). fp16 operands carry W as an exact
// hi + lo pair (W = W_hi + W_lo + O(2^-22 |W|)); x is fp16 already, so both
// products are exact and only the fp32 accumulation rounds.
//
//   [Y_hi | Y_lo] = X [W_hi ; W_lo]^T as one N = 256 product per K step of 16 (the
//   X tile is read once per K step), Y = Y_hi + Y_lo in the epilogue. An MMA has
//   N <= 256, so a CTA produces 128 channels:
//   D = 128: one CTA per tile, all channels, K = 128;
//   D = 256: two CTAs per tile (a CTA pair walks the same tiles), each with one
//            half of the channels and its half of W resident (128 KB), K = 256;
//            the pair's second read of each X tile is served by L2.
//
// Roles (one CTA per SM, persistent over a contiguous range of tiles):
//   warp 0      TMA producer: the plan's W (resident, reloaded when the job
//               changes) and a ring of ten 16 KB K-chunks of X tiles (128-byte
//               swizzle), each freed as soon as the MMAs reading it complete;
//   warp 1      TMEM allocation and the single MMA-issuing thread;
//   warps 2-9   epilogue: one thread per (vector, half of the channel groups);
//               two warps per TMEM lane quarter; 32 columns per tcgen05.ld,
//               group abs-max, fp16 scale, int4 rounding, nibble packing,
//               16-byte code stores and one scale store per half vector.
// Two TMEM accumulators (2 x D columns) let the epilogue of tile i overlap the
// MMAs of tile i + 1. Every wait is bounded; a CTA that gives up raises a device
// error flag and still deallocates its TMEM.
//
// Exact W (EX, plans of the SRHT variant): W = H diag(s) has entries +-1, exact in
// fp16, so one product per K step gives Y exactly up to the fp32 accumulation; the
// per-channel factor lambda_c / sqrt(D) is applied in the epilogue. An MMA then
// covers all D channels (N = D), one CTA per tile at either head dim, half the
// tensor work of the hi/lo product.
#include <algorithm>
#include <cstdio>
#include <mutex>

#include "kvq_internal.h"
#include "kvq_ptx.cuh"
#include "kvq_quant.cuh"

namespace kvq {

__device__ uint32_t g_enc_tc_err = 0;

namespace {

constexpr int kTcRows = 128;    // vectors per tile (MMA M)

constexpr int kTcEpiWarps = 8;  // two per TMEM lane quarter, each taking half the channel groups
constexpr int kTcThreads = 32 * (2 + kTcEpiWarps);
constexpr int kTcMaxJobs = 64;

struct alignas(64) TcJob {
  CUtensorMap xmap;  // x as [rows][D] fp16, box {64, 128}, 128-byte swizzle
  CUtensorMap wmap;  // W as [2D][D] fp16 (hi rows, then lo rows; EX: [D][D]), box {64, N}, 128-byte swizzle
  uint8_t* codes;    // [BH][T_cap][D * BITS / 8]
  uint16_t* scales;  // [BH][T_cap][D/G]
  const float* chan; // EX: the per-channel factors lambda_c / sqrt(D)
  int rows, n, T_cap, pos, tile0;  // rows = B*H*n; tile0 = first global tile of the job
};

template <int MAXJ>
struct TcBatch {
  TcJob j[MAXJ];
  int njobs, ntiles;
};

template <int D, bool EX>
struct TcCfg {
  static constexpr int KC = D / 64;                  // 64-wide K chunks (one 128-byte swizzle atom each)
  static constexpr int kSplit = EX ? 1 : D / 128;    // CTAs per tile (channel halves)
  static constexpr int kChunkA = kTcRows * 128;      // one K chunk of a 128-row X tile: 16 KB
  static constexpr int kN = EX ? D : 256;            // MMA N: D exact rows, or 128 W_hi rows then 128 W_lo rows
  static constexpr int kChunkW = kN * 128;           // one K chunk of W
  static constexpr int kW = KC * kChunkW;            // 64 KB (D = 128) or 128 KB (D = 256); EX: 32 / 128 KB
  static constexpr int kChunks = (EX && D == 128) ? 12 : (D == 128 ? 10 : 6);  // X ring depth in K chunks
  static constexpr int kTmemCols = 2 * kN;           // two accumulators of N fp32 columns
  static constexpr int kBars = 8 * (2 * kChunks + 4 + 3) + 16;
  static constexpr int kSmem = kW + kChunks * kChunkA + kBars + 1024;
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ int job_of(const TcJob* jobs, int njobs, int job, int t) {
  while (job + 1 < njobs && jobs[job + 1].tile0 <= t) ++job;
  return job;
}

// The quantiser over one 32-channel chunk: one group of 32 or two of 16 (sb: their
// scales); BITS code words (the chunk's 16 or 32 code bytes).
template <int G, int BITS>
__device__ __forceinline__ void quantize_chunk(const float (&y)[32], uint32_t (&w)[BITS], uint32_t (&sb)[32 / G]) {
  if constexpr (G == 32) {
    quantize_group<32, BITS>(y, w, sb[0]);
  } else {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float yh[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) yh[i] = y[16 * j + i];
      uint32_t wh[BITS / 2];
      quantize_group<16, BITS>(yh, wh, sb[j]);
#pragma unroll
      for (int i = 0; i < BITS / 2; ++i) w[(BITS / 2) * j + i] = wh[i];
    }
  }
}

// the code bytes of 32-channel chunk k of cache row `orow` (16 or 32 bytes)
template <int D, int BITS>
__device__ __forceinline__ void store_chunk(uint8_t* codes, size_t orow, int k, const uint32_t (&w)[BITS]) {
  uint4* row = reinterpret_cast<uint4*>(codes + orow * (D * BITS / 8));
  if constexpr (BITS == 4) {
    row[k] = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
    row[2 * k] = make_uint4(w[0], w[1], w[2], w[3]);
    row[2 * k + 1] = make_uint4(w[4], w[5], w[6], w[7]);
  }
}

// n consecutive fp16 scale bits (n = 2, 4 or 8) to one 4-, 8- or 16-byte store
template <int N>
__device__ __forceinline__ void store_scales(uint16_t* dst, const uint32_t (&sb)[N]) {
  static_assert(N == 2 || N == 4 || N == 8, "scale count");
  if constexpr (N == 2) {
    *reinterpret_cast<uint32_t*>(dst) = sb[0] | (sb[1] << 16);
  } else if constexpr (N == 4) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(sb[0] | (sb[1] << 16), sb[2] | (sb[3] << 16));
  } else {
    *reinterpret_cast<uint4*>(dst) = make_uint4(sb[0] | (sb[1] << 16), sb[2] | (sb[3] << 16), sb[4] | (sb[5] << 16),
                                                sb[6] | (sb[7] << 16));
  }
}

template <int D, bool EX, int G, int BITS, int MAXJ>
__global__ void __launch_bounds__(kTcThreads, 1) encode_tc_kernel(const __grid_constant__ TcBatch<MAXJ> bt) {
  using C = TcCfg<D, EX>;
  constexpr int kTcChunks = C::kChunks;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sW = sm;
  uint8_t* sA = sm + C::kW;
  uint64_t* afull = reinterpret_cast<uint64_t*>(sA + kTcChunks * C::kChunkA);
  uint64_t* aempty = afull + kTcChunks;
  uint64_t* tfull = aempty + kTcChunks;
  uint64_t* tempty = tfull + 2;
  uint64_t* wfull = tempty + 2;
  uint64_t* wempty = wfull + 1;
  uint64_t* mdone = wempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mdone + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // D = 256: CTAs 2p and 2p + 1 take the same tiles, channel halves 0 and 1
  const int half = C::kSplit == 2 ? (int)(blockIdx.x & 1) : 0;
  const int nwalk = (int)gridDim.x / C::kSplit, walker = (int)blockIdx.x / C::kSplit;
  const int per = (bt.ntiles + nwalk - 1) / nwalk;
  const int t_begin = walker * per;
  const int t_end = min(t_begin + per, bt.ntiles);
  const int ntile = max(0, t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcChunks; ++s) {
      mbar_init(&afull[s], 1);
      mbar_init(&aempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kTcEpiWarps);  // one arrival per epilogue warp
    }
    mbar_init(wfull, 1);
    mbar_init(wempty, 1);
    mbar_init(mdone, 1);
    fence_mbarrier_init();
  }
  // programmatic dependent launch: the next kernel in the stream may start its own
  // prologue now (it reads what this kernel writes only after its grid dependency wait)
  grid_dep_launch();
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && ntile > 0) {
      const uint64_t pol = l2_evict_first_policy();
      int job = job_of(bt.j, bt.njobs, 0, t_begin), wjob = -1, nw = 0;
      // the first job's W (a plan constant, written once when the plan is made) is
      // loaded while the previous kernel in the stream finishes; the inputs after it
      mbar_arrive_expect_tx(wfull, C::kW);
#pragma unroll
      for (int kc = 0; kc < C::KC; ++kc) tma_load_2d(sW + kc * C::kChunkW, &bt.j[job].wmap, wfull, kc * 64, 256 * half);
      wjob = job;
      nw = 1;
      grid_dep_wait();
      for (int i = 0; i < ntile; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        const TcJob& J = bt.j[job];
        if (job != wjob) {
          if (nw > 0 && !mbar_wait_bounded(wempty, (nw - 1) & 1)) {
            atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
            break;
          }
          mbar_arrive_expect_tx(wfull, C::kW);
#pragma unroll
          for (int kc = 0; kc < C::KC; ++kc) tma_load_2d(sW + kc * C::kChunkW, &J.wmap, wfull, kc * 64, 256 * half);
          wjob = job;
          ++nw;
        }
        // the tile's K chunks, each into the next slot of the chunk ring
        const int row = (t - J.tile0) * kTcRows;
        bool ok = true;
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc) {
          const int c = i * C::KC + kc, s = c % kTcChunks;
          if (c >= kTcChunks && !mbar_wait_bounded(&aempty[s], ((c / kTcChunks) - 1) & 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&afull[s], C::kChunkA);
          tma_load_2d_hint(sA + s * C::kChunkA, &J.xmap, &afull[s], kc * 64, row, pol);
        }
        if (!ok) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && ntile > 0) {
      constexpr uint32_t idesc = umma_idesc_f16(kTcRows, C::kN);
      int job = job_of(bt.j, bt.njobs, 0, t_begin), wjob = -1, nw = 0;
      for (int i = 0; i < ntile; ++i) {
        const int t = t_begin + i;
        job = job_of(bt.j, bt.njobs, job, t);
        if (job != wjob) {
          if (nw > 0) umma_commit(wempty);  // W may be replaced once the MMAs issued so far are done
          if (!mbar_wait_bounded(wfull, nw & 1)) {
            atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
            break;
          }
          wjob = job;
          ++nw;
        }
        const int a = i & 1;
        if (i >= 2 && !mbar_wait_bounded(&tempty[a], ((i >> 1) - 1) & 1)) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(a * C::kN);
        const uint32_t w0 = smem_u32(sW);
        bool ok = true;
#pragma unroll
        for (int kc = 0; kc < C::KC; ++kc) {
          const int c = i * C::KC + kc, s = c % kTcChunks;
          if (!mbar_wait_bounded(&afull[s], (c / kTcChunks) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * C::kChunkA);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // K = 16 per MMA: 32 bytes along the swizzled row
            const uint64_t ad = umma_desc_sw128(a0 + kk * 32);
            const uint64_t wd = umma_desc_sw128(w0 + kc * C::kChunkW + kk * 32);
            umma_f16(d, ad, wd, idesc, (kc | kk) != 0);
          }
          umma_commit(&aempty[s]);  // this chunk is free once these MMAs have read it
        }
        if (!ok) {
          atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
          break;
        }
        umma_commit(&tfull[a]);  // the accumulator is ready for the epilogue
      }
      // TMEM is released below: wait (bounded) until every MMA of this CTA has completed
      // (a commit with nothing outstanding arrives at once)
      umma_commit(mdone);
      if (!mbar_wait_bounded(mdone, 0)) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w: TMEM lanes 32 (w % 4) .. + 31 (one vector per thread), channel groups
    // [h * NGH, (h + 1) * NGH) of the CTA's channels with h = (w - 2) / 4
    constexpr int NGH = EX ? D / 64 : 2;  // 32-channel chunks per thread: two threads per vector
    constexpr int SPC = 32 / G;            // scale groups per chunk
    const int q = warp & 3;
    const int h = (warp - 2) >> 2;
    int job = ntile > 0 ? job_of(bt.j, bt.njobs, 0, t_begin) : 0;
    for (int i = 0; i < ntile; ++i) {
      const int t = t_begin + i;
      job = job_of(bt.j, bt.njobs, job, t);
      const TcJob& J = bt.j[job];
      const int a = i & 1;
      // warp-uniform outcome: the tcgen05.ld below needs the whole warp
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&tfull[a], (i >> 1) & 1))) {
        if (lane == 0) atomicOr(&g_enc_tc_err, kErrTimeoutLoad);
        break;
      }
      tc_fence_after();
      const int r = (t - J.tile0) * kTcRows + 32 * q + lane;  // row of this thread's vector in the job
      const bool valid = r < J.rows;
      const int bh = valid ? r / J.n : 0;
      const size_t orow = (size_t)bh * J.T_cap + J.pos + (r - bh * J.n);
      const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(a * C::kN + 32 * NGH * h);
      uint32_t sb[NGH * SPC];
      if constexpr (EX) {
        // Y exact up to the fp32 accumulation; y = Y * lambda_c / sqrt(D)
        float y[NGH][32];
#pragma unroll
        for (int g = 0; g < NGH; ++g) tmem_ld32(ta + 32 * g, y[g]);
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < NGH; ++g) tmem_regs_fence(y[g]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
          const float4* f4 = reinterpret_cast<const float4*>(J.chan + 32 * (NGH * h + g));
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 f = __ldg(f4 + e);
            y[g][4 * e] *= f.x;
            y[g][4 * e + 1] *= f.y;
            y[g][4 * e + 2] *= f.z;
            y[g][4 * e + 3] *= f.w;
          }
          uint32_t w[BITS], sg[SPC];
          quantize_chunk<G, BITS>(y[g], w, sg);
#pragma unroll
          for (int j = 0; j < SPC; ++j) sb[SPC * g + j] = sg[j];
          if (valid) store_chunk<D, BITS>(J.codes, orow, NGH * h + g, w);
        }
        if (valid) store_scales<NGH * SPC>(J.scales + orow * (D / G) + NGH * SPC * h, sb);
      } else {
        float y[NGH][32], ylo[NGH][32];
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
          tmem_ld32(ta + 32 * g, y[g]);
          tmem_ld32(ta + 128 + 32 * g, ylo[g]);
        }
        tmem_ld_wait();
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
          tmem_regs_fence(y[g]);
          tmem_regs_fence(ylo[g]);
        }
        // the accumulator may be overwritten as soon as every epilogue warp has its values
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[a]);
#pragma unroll
        for (int g = 0; g < NGH; ++g) {
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 v = __fadd2_rn(make_float2(y[g][e], y[g][e + 1]), make_float2(ylo[g][e], ylo[g][e + 1]));
            y[g][e] = v.x;
            y[g][e + 1] = v.y;
          }
          uint32_t w[BITS], sg[SPC];
          quantize_chunk<G, BITS>(y[g], w, sg);
#pragma unroll
          for (int j = 0; j < SPC; ++j) sb[SPC * g + j] = sg[j];
          if (valid) store_chunk<D, BITS>(J.codes, orow, 4 * half + NGH * h + g, w);
        }
        if (valid) store_scales<NGH * SPC>(J.scales + orow * (D / G) + SPC * (4 * half + NGH * h), sb);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}


void tc_prepare() {
  static std::once_flag once;
  std::call_once(once, [] {
    for (int bits : {4, 8})
      for (int D : {128, 256})
        for (int G : {32, 16})
          dispatch_dgb(D, G, bits, [](auto d, auto g, auto b) {
            constexpr int kD = decltype(d)::value, kG = decltype(g)::value, kB = decltype(b)::value;
            cudaFuncSetAttribute(encode_tc_kernel<kD, false, kG, kB, kTcMaxJobs>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<kD, false>::kSmem);
            cudaFuncSetAttribute(encode_tc_kernel<kD, true, kG, kB, kTcMaxJobs>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<kD, true>::kSmem);
            return 0;
          });
  });
}

template <int D, bool EX, int G, int BITS>
cudaError_t tc_launch(cudaLaunchConfig_t cfg, const TcBatch<kTcMaxJobs>& bt, int tiles, int sms) {
  cfg.gridDim = dim3(TcCfg<D, EX>::kSplit == 2 ? 2 * std::min(tiles, sms / 2) : std::min(tiles, sms));
  cfg.dynamicSmemBytes = TcCfg<D, EX>::kSmem;
  return cudaLaunchKernelEx(&cfg, encode_tc_kernel<D, EX, G, BITS, kTcMaxJobs>, bt);
}

}  // namespace

bool encode_tc_supported(int D, int G) { return (D == 128 || D == 256) && (G == 32 || G == 16); }

// Grouped launch over jobs of one head_dim (128 or 256), group (32 or 16), transform and
// code width (4 or 8 bits); jobs with no rows are skipped.
kvq_status launch_encode_tc(const kvq_encode_job* jobs, int njobs, cudaStream_t strm) {
  const int D = jobs[0].plan->D;
  const bool ex = jobs[0].plan->xform == 1;  // SRHT: exact W
  tc_prepare();
  int i0 = 0;
  while (i0 < njobs) {
    TcBatch<kTcMaxJobs> bt{};
    int nj = 0, tiles = 0;
    int i = i0;
    for (; i < njobs && nj < kTcMaxJobs; ++i) {
      const kvq_encode_job& j = jobs[i];
      const long rows = (long)j.B * j.H * j.n;
      if (rows == 0) continue;
      if (rows > (1l << 31) - 1) return fail(KVQ_ERR_UNSUPPORTED, "encode: more than 2^31 - 1 vectors in one job");
      TcJob& J = bt.j[nj];
      const uint64_t xd[2] = {(uint64_t)D, (uint64_t)rows};
      const uint64_t xs[1] = {(uint64_t)D * 2};
      const uint32_t xb[2] = {64u, (uint32_t)kTcRows};
      kvq_status st = encode_tiled(&J.xmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, j.x, xd, xs, xb,
                                   CU_TENSOR_MAP_SWIZZLE_128B, "encode x");
      if (st != KVQ_OK) return st;
      // W = Lambda F_r diag(s): per 128-channel half, 128 hi rows then 128 lo rows, D
      // columns; exact W (SRHT): H diag(s), D rows (channels), D columns
      const uint64_t wd[2] = {(uint64_t)D, (uint64_t)(ex ? D : 2 * D)};
      const uint64_t ws[1] = {(uint64_t)D * 2};
      const uint32_t wb[2] = {64u, (uint32_t)(ex ? D : 256)};
      st = encode_tiled(&J.wmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, j.plan->wt_dev, wd, ws, wb,
                        CU_TENSOR_MAP_SWIZZLE_128B, "encode weights");
      if (st != KVQ_OK) return st;
      J.codes = j.codes;
      J.scales = j.scales;
      J.chan = j.plan->enc_dev->chan;
      J.rows = (int)rows;
      J.n = j.n;
      J.T_cap = j.T_cap;
      J.pos = j.pos;
      J.tile0 = tiles;
      tiles += (int)((rows + kTcRows - 1) / kTcRows);
      ++nj;
    }
    i0 = i;
    if (nj == 0) continue;
    bt.njobs = nj;
    bt.ntiles = tiles;
    int dev = 0;
    cudaGetDevice(&dev);
    const int sms = num_sms(dev);
    // programmatic dependent launch: the kernel loads its first W and allocates TMEM
    // while the previous kernel in the stream finishes (grid dependency wait before the
    // inputs and every global write)
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(kTcThreads);
    cfg.stream = strm;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = dispatch_dgb(D, jobs[0].plan->G, jobs[0].plan->bits, [&](auto d, auto g, auto b) {
      constexpr int kD = decltype(d)::value, kG = decltype(g)::value, kB = decltype(b)::value;
      return ex ? tc_launch<kD, true, kG, kB>(cfg, bt, tiles, sms) : tc_launch<kD, false, kG, kB>(cfg, bt, tiles, sms);
    });
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return fail(KVQ_ERR_CUDA, std::string("encode (tensor cores) launch: ") + cudaGetErrorString(e));
  }
  return KVQ_OK;
}

uint32_t encode_tc_error_flags(bool clear) {
  uint32_t v = 0;
  cudaMemcpyFromSymbol(&v, g_enc_tc_err, sizeof(v));
  if (clear && v) {
    const uint32_t z = 0;
    cudaMemcpyToSymbol(g_enc_tc_err, &z, sizeof(z));
  }
  return v;
}

}  // namespace kvq
