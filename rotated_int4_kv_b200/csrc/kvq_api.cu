// kvq_api.cu -- the C ABI: plan management, host-side argument checks, error
// reporting and the driver entry point for TMA tensor maps.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>
#include <vector>

#include "kvq_internal.h"

namespace kvq {

uint32_t codec_error_flags(bool clear);
uint32_t attend_error_flags(bool clear);

namespace {
thread_local std::string t_last_error;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Per-channel normalisation of the real basis: dg_c = 1/sqrt(D) (DC, Nyquist),
// sqrt(2/D) (cos rows), -sqrt(2/D) (sin rows: the spectrum slot holds Im X_k and
// the sin row equals -sqrt(2/D) Im X_k).
// Row c of the orthonormal real basis in channel order, at sample n: DC, then
// (cos_k, +sin_k) pairs, then Nyquist; angles from the exact residue k n mod D.
double basis_value(int c, int n, int D) {
  const double pi2 = 6.283185307179586476925286766559;
  if (c == 0) return 1.0 / std::sqrt((double)D);
  if (c == D - 1) return ((n & 1) ? -1.0 : 1.0) / std::sqrt((double)D);
  const int k = (c + 1) / 2;
  const double ang = pi2 * (double)((long)k * n % D) / (double)D;
  return std::sqrt(2.0 / D) * ((c & 1) ? std::cos(ang) : std::sin(ang));
}

// Entry (i, j) of the Sylvester Hadamard matrix in natural order: (-1)^popcount(i & j).
double hadamard_value(int i, int j) { return (__builtin_popcount((unsigned)(i & j)) & 1) ? -1.0 : 1.0; }

uint16_t half_bits(float f) { return __half_as_ushort(__float2half_rn(f)); }
float half_value(uint16_t b) { return __half2float(__ushort_as_half(b)); }

double basis_dg(int c, int D) {
  if (c == 0 || c == D - 1) return 1.0 / std::sqrt((double)D);
  return (c & 1) ? std::sqrt(2.0 / D) : -std::sqrt(2.0 / D);
}

}  // namespace

void set_error(const std::string& msg) { t_last_error = msg; }

kvq_status fail(kvq_status st, const std::string& msg) {
  t_last_error = msg;
  return st;
}

std::atomic<int> g_encode_path{0};

int encode_path() { return g_encode_path.load(); }

std::atomic<int> g_decode_path{0};

int decode_path() { return g_decode_path.load(); }

// All jobs share head_dim and group (checked by the callers).
kvq_status dispatch_encode(const kvq_encode_job* jobs, int njobs, cudaStream_t s) {
  const kvq_plan* p = jobs[0].plan;
  const int path = g_encode_path.load();
  const bool tc = encode_tc_supported(p->D, p->G) && p->wt_dev != nullptr;
  if (path == 2 && !tc)
    return fail(KVQ_ERR_UNSUPPORTED, "encode: the tensor-core path supports head_dim 128 or 256 with group 32 or 16");
  if (path == 3) {
    if (!encode_split_supported(p))
      return fail(KVQ_ERR_UNSUPPORTED, "encode: the radix-2 split path serves head_dim 256 SRFT plans");
    return launch_encode_tc(jobs, njobs, s, true);
  }
  if (tc && path != 1) return launch_encode_tc(jobs, njobs, s, false);
  return launch_encode_jobs(jobs, njobs, s);
}

namespace {
// Small cache of encoded tensor maps: repeated calls on the same buffers (the
// usual decode loop) skip the driver call. Keyed by every encoding input.
struct MapKey {
  uint64_t w[20];
  bool operator==(const MapKey& o) const { return std::memcmp(w, o.w, sizeof(w)) == 0; }
};
struct MapKeyHash {
  size_t operator()(const MapKey& k) const {
    uint64_t h = 1469598103934665603ull;
    for (uint64_t v : k.w) h = (h ^ v) * 1099511628211ull;
    return (size_t)h;
  }
};
std::mutex g_map_mu;
std::unordered_map<MapKey, CUtensorMap, MapKeyHash> g_maps;
constexpr size_t kMaxCachedMaps = 8192;
}  // namespace

kvq_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base, const uint64_t* dims,
                        const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz,
                        const char* what) {
  MapKey key{};
  key.w[0] = (uint64_t)dt | ((uint64_t)rank << 8) | ((uint64_t)swz << 16);
  key.w[1] = reinterpret_cast<uint64_t>(base);
  for (int i = 0; i < rank && i < 5; ++i) {
    key.w[2 + i] = dims[i];
    key.w[7 + i] = box[i];
  }
  for (int i = 0; i + 1 < rank && i < 4; ++i) key.w[12 + i] = strides_bytes[i];
  int dev = -1;
  cudaGetDevice(&dev);
  key.w[16] = (uint64_t)(int64_t)dev;
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    auto it = g_maps.find(key);
    if (it != g_maps.end()) {
      *map = it->second;
      return KVQ_OK;
    }
  }
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return fail(KVQ_ERR_CUDA, "cuTensorMapEncodeTiled not available from the driver");
  cuuint64_t d[5];
  cuuint64_t st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
  const CUresult r = fn(map, dt, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(KVQ_ERR_CUDA, std::string("tensor map for ") + what + " rejected by the driver");
  std::lock_guard<std::mutex> lk(g_map_mu);
  if (g_maps.size() >= kMaxCachedMaps) g_maps.clear();
  g_maps.emplace(key, *map);
  return KVQ_OK;
}

int num_sms(int device) {
  static int cache[64] = {0};
  if (device < 0 || device >= 64) return 148;
  if (cache[device] == 0) {
    int v = 0;
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, device);
    cache[device] = v > 0 ? v : 148;
  }
  return cache[device];
}

kvq_status check_plan_device(const kvq_plan* p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(KVQ_ERR_DEVICE, "no current CUDA device");
  if (dev != p->device) return fail(KVQ_ERR_DEVICE, "plan belongs to another device");
  return KVQ_OK;
}

}  // namespace kvq

using kvq::fail;

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_ALIGNMENT: return "misaligned pointer or size";
    case KVQ_ERR_CAPACITY: return "cache capacity exceeded";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_DEVICE: return "device mismatch or unsupported device";
  }
  return "unknown status";
}

const char* kvq_last_error(void) { return kvq::t_last_error.c_str(); }

kvq_status kvq_plan_create(kvq_plan** out, int D, int G, const int8_t* signs, const float* lambda) {
  return kvq_plan_create_transform(out, D, G, signs, lambda, KVQ_TRANSFORM_SRFT);
}

int kvq_plan_transform(const kvq_plan* p) { return p ? p->xform : -1; }

int kvq_plan_bits(const kvq_plan* p) { return p ? p->bits : -1; }

kvq_status kvq_plan_create_transform(kvq_plan** out, int D, int G, const int8_t* signs, const float* lambda,
                                     int transform) {
  return kvq_plan_create_ex(out, D, G, signs, lambda, transform, 4);
}

kvq_status kvq_plan_create_ex(kvq_plan** out, int D, int G, const int8_t* signs, const float* lambda, int transform,
                              int bits) {
  if (!out || !signs || !lambda) return fail(KVQ_ERR_INVALID_ARG, "plan_create: null argument");
  *out = nullptr;
  if (bits != 4 && bits != 8) return fail(KVQ_ERR_UNSUPPORTED, "plan_create: bits must be 4 or 8");
  if (transform != KVQ_TRANSFORM_SRFT && transform != KVQ_TRANSFORM_SRHT)
    return fail(KVQ_ERR_UNSUPPORTED, "plan_create: transform must be KVQ_TRANSFORM_SRFT or KVQ_TRANSFORM_SRHT");
  const bool hadamard = transform == KVQ_TRANSFORM_SRHT;
  if (D != 128 && D != 256) return fail(KVQ_ERR_UNSUPPORTED, "plan_create: head_dim must be 128 or 256");
  if (G != 32 && G != 16) return fail(KVQ_ERR_UNSUPPORTED, "plan_create: group must be 32 or 16");
  for (int i = 0; i < D; ++i) {
    if (signs[i] != 1 && signs[i] != -1) return fail(KVQ_ERR_INVALID_ARG, "plan_create: signs must be +1/-1");
    if (!(std::isfinite(lambda[i]) && lambda[i] > 0.0f))
      return fail(KVQ_ERR_INVALID_ARG, "plan_create: lambda must be finite and > 0");
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(KVQ_ERR_DEVICE, "plan_create: no CUDA device");
  cudaDeviceProp prop{};
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10)
    return fail(KVQ_ERR_DEVICE, "plan_create: needs a compute capability 10.x (sm_100) device");

  kvq_plan* p = new kvq_plan();
  p->D = D;
  p->G = G;
  p->device = dev;
  p->xform = transform;
  p->bits = bits;
  // per-channel factor of the rotation's unnormalised rows: the real DFT's dg_c, or
  // 1/sqrt(D) for every Hadamard row
  for (int c = 0; c < D; ++c) {
    const double dg = hadamard ? 1.0 / std::sqrt((double)D) : kvq::basis_dg(c, D);
    p->enc.chan[c] = (float)((double)lambda[c] * dg);
    p->dec.chan[c] = (float)(dg / (double)lambda[c]);
  }
  for (int w = 0; w < D / 2; ++w) {
    const uint32_t m = (signs[2 * w] < 0 ? 0x8000u : 0u) | (signs[2 * w + 1] < 0 ? 0x80000000u : 0u);
    p->enc.sgn[w] = m;
    p->dec.sgn[w] = m;
  }
  // tensor-core encode operand: W = Lambda F_r diag(s) (channel rows, D columns) as an
  // fp16 pair (value = hi + lo to ~2^-22 |W|), laid out per 128-channel half h as
  // 128 hi rows then 128 lo rows: row 256 h + r = hi of channel 128 h + r,
  // row 256 h + 128 + r = lo of the same channel.
  // SRHT plans: W = H diag(s) exactly (entries +-1; D rows, D columns), the factor
  // lambda_c / sqrt(D) is applied by the kernel's epilogue.
  std::vector<uint16_t> wt(hadamard ? (size_t)D * D : (size_t)2 * D * D);
  for (int c = 0; c < D; ++c) {
    const int h = c / 128, rr = c % 128;
    for (int n = 0; n < D; ++n) {
      if (hadamard) {
        wt[(size_t)c * D + n] = kvq::half_bits((float)(kvq::hadamard_value(c, n) * (double)signs[n]));
        continue;
      }
      const double w = (double)lambda[c] * kvq::basis_value(c, n, D) * (double)signs[n];
      const uint16_t hi = kvq::half_bits((float)w);
      const uint16_t lo = kvq::half_bits((float)(w - (double)kvq::half_value(hi)));
      wt[(size_t)(256 * h + rr) * D + n] = hi;
      wt[(size_t)(256 * h + 128 + rr) * D + n] = lo;
    }
  }
  // attention operand (both head dims): the unnormalised 128-point real DFT in slot
  // order, F128 (hi, lo): row 0 = 1, row 1 = (-1)^m, row 2k = cos(2 pi k m / 128),
  // row 2k+1 = -sin(2 pi k m / 128); for the SRHT the 128-point Hadamard matrix (exact
  // in fp16, lo = 0). D = 128 applies it directly, D = 256 to the even and odd samples;
  // the plan's signs and per-channel factors are applied around it.
  std::vector<uint16_t> rot;
  {
    const int M = 128;
    rot.resize((size_t)2 * M * M);
    const double pi2 = 6.283185307179586476925286766559;
    for (int j = 0; j < M; ++j)
      for (int m = 0; m < M; ++m) {
        double v;
        if (hadamard) v = kvq::hadamard_value(j, m);
        else if (j == 0) v = 1.0;
        else if (j == 1) v = (m & 1) ? -1.0 : 1.0;
        else {
          const double ang = pi2 * (double)((long)(j / 2) * m % M) / (double)M;
          v = (j & 1) ? -std::sin(ang) : std::cos(ang);
        }
        const uint16_t hi = kvq::half_bits((float)v);
        const uint16_t lo = kvq::half_bits((float)(v - (double)kvq::half_value(hi)));
        rot[(size_t)j * M + m] = hi;
        rot[(size_t)(M + j) * M + m] = lo;
      }
  }
  // tensor-core decode operand: W_dec = diag(s) Q^T Lambda^-1 (row n = output sample n,
  // column = channel), one fp16 rounding per entry; the columns of each 16-byte unit in
  // the order the kernel's dequantiser writes the channels (decode_unit_channel)
  std::vector<uint16_t> wdec((size_t)D * D);
  for (int n = 0; n < D; ++n)
    for (int k = 0; k < D; ++k) {
      const int c = (k & ~7) + kvq::decode_unit_channel(k & 7, bits);
      const double q = hadamard ? kvq::hadamard_value(c, n) / std::sqrt((double)D) : kvq::basis_value(c, n, D);
      wdec[(size_t)n * D + k] = kvq::half_bits((float)((double)signs[n] * q / (double)lambda[c]));
    }
  constexpr size_t kWtOff = 4096;  // after the two CodecConsts copies, 16-byte aligned for TMA
  static_assert(2 * sizeof(kvq::CodecConsts) <= kWtOff, "plan block layout");
  const size_t rot_off = kWtOff + wt.size() * 2;
  const size_t wdec_off = rot_off + rot.size() * 2;
  const size_t bytes = wdec_off + wdec.size() * 2;
  void* blk = nullptr;
  if (cudaMalloc(&blk, bytes) != cudaSuccess) {
    delete p;
    return fail(KVQ_ERR_CUDA, "plan_create: cudaMalloc failed");
  }
  if (cudaMemcpy(blk, &p->enc, sizeof(kvq::CodecConsts), cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy((char*)blk + sizeof(kvq::CodecConsts), &p->dec, sizeof(kvq::CodecConsts), cudaMemcpyHostToDevice) !=
          cudaSuccess ||
      (!wt.empty() &&
       cudaMemcpy((char*)blk + kWtOff, wt.data(), wt.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) ||
      (!rot.empty() &&
       cudaMemcpy((char*)blk + rot_off, rot.data(), rot.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) ||
      cudaMemcpy((char*)blk + wdec_off, wdec.data(), wdec.size() * 2, cudaMemcpyHostToDevice) != cudaSuccess) {
    cudaFree(blk);
    delete p;
    return fail(KVQ_ERR_CUDA, "plan_create: upload failed");
  }
  p->dblock = blk;
  p->enc_dev = reinterpret_cast<const kvq::CodecConsts*>(blk);
  p->dec_dev = reinterpret_cast<const kvq::CodecConsts*>((char*)blk + sizeof(kvq::CodecConsts));
  p->wt_dev = wt.empty() ? nullptr : reinterpret_cast<const uint16_t*>((char*)blk + kWtOff);
  p->rot_dev = reinterpret_cast<const uint16_t*>((char*)blk + rot_off);
  p->wdec_dev = reinterpret_cast<const uint16_t*>((char*)blk + wdec_off);
  *out = p;
  return KVQ_OK;
}

kvq_status kvq_plan_destroy(kvq_plan* p) {
  if (!p) return KVQ_OK;
  if (p->dblock) {
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != p->device) cudaSetDevice(p->device);
    cudaFree(p->dblock);
    if (cur != p->device && cur >= 0) cudaSetDevice(cur);
  }
  delete p;
  return KVQ_OK;
}

int kvq_plan_head_dim(const kvq_plan* p) { return p ? p->D : -1; }
int kvq_plan_group(const kvq_plan* p) { return p ? p->G : -1; }

kvq_status kvq_encode(const kvq_plan* p, const uint16_t* x, int B, int H, int n, uint8_t* codes, uint16_t* scales,
                      int T_cap, int pos, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "encode: null plan");
  if (B < 0 || H < 0 || n < 0 || T_cap < 0 || pos < 0) return fail(KVQ_ERR_INVALID_ARG, "encode: negative size");
  if ((long)pos + n > T_cap) return fail(KVQ_ERR_CAPACITY, "encode: pos + n > T_cap");
  if (B == 0 || H == 0 || n == 0) return KVQ_OK;
  if (!x || !codes || !scales) return fail(KVQ_ERR_INVALID_ARG, "encode: null buffer");
  if (!kvq::aligned16(x) || !kvq::aligned16(codes) || !kvq::aligned16(scales))
    return fail(KVQ_ERR_ALIGNMENT, "encode: buffers must be 16-byte aligned");
  if ((long)B * H > (1L << 30) || (long)T_cap * B * H > (1L << 40)) return fail(KVQ_ERR_INVALID_ARG, "encode: too large");
  kvq_status st = kvq::check_plan_device(p);
  if (st != KVQ_OK) return st;
  kvq_encode_job job{p, x, codes, scales, B, H, n, T_cap, pos};
  return kvq::dispatch_encode(&job, 1, (cudaStream_t)stream);
}

kvq_status kvq_encode_batch(const kvq_encode_job* jobs, int njobs, void* stream) {
  if (njobs < 0 || (njobs > 0 && !jobs)) return fail(KVQ_ERR_INVALID_ARG, "encode_batch: bad job array");
  std::vector<kvq_encode_job> live;
  live.reserve(njobs);
  const kvq_plan* p0 = nullptr;
  for (int i = 0; i < njobs; ++i) {
    const kvq_encode_job& j = jobs[i];
    const std::string w = "encode_batch job " + std::to_string(i) + ": ";
    if (!j.plan) return fail(KVQ_ERR_INVALID_ARG, w + "null plan");
    if (j.B < 0 || j.H < 0 || j.n < 0 || j.T_cap < 0 || j.pos < 0) return fail(KVQ_ERR_INVALID_ARG, w + "negative size");
    if ((long)j.pos + j.n > j.T_cap) return fail(KVQ_ERR_CAPACITY, w + "pos + n > T_cap");
    if (j.B == 0 || j.H == 0 || j.n == 0) continue;
    if (!j.x || !j.codes || !j.scales) return fail(KVQ_ERR_INVALID_ARG, w + "null buffer");
    if (!kvq::aligned16(j.x) || !kvq::aligned16(j.codes) || !kvq::aligned16(j.scales))
      return fail(KVQ_ERR_ALIGNMENT, w + "buffers must be 16-byte aligned");
    if ((long)j.B * j.H > (1L << 30) || (long)j.T_cap * j.B * j.H > (1L << 40)) return fail(KVQ_ERR_INVALID_ARG, w + "too large");
    if (!p0) {
      p0 = j.plan;
      kvq_status st = kvq::check_plan_device(p0);
      if (st != KVQ_OK) return st;
    } else if (j.plan->D != p0->D || j.plan->G != p0->G || j.plan->device != p0->device ||
               j.plan->xform != p0->xform || j.plan->bits != p0->bits) {
      return fail(KVQ_ERR_INVALID_ARG, w + "all jobs must share head_dim, group, transform, code width and device");
    }
    live.push_back(j);
  }
  if (live.empty()) return KVQ_OK;
  return kvq::dispatch_encode(live.data(), (int)live.size(), (cudaStream_t)stream);
}

kvq_status kvq_set_encode_path(int path) {
  if (path < 0 || path > 3) return fail(KVQ_ERR_INVALID_ARG, "set_encode_path: path must be 0, 1, 2 or 3");
  kvq::g_encode_path.store(path);
  return KVQ_OK;
}

int kvq_get_encode_path(void) { return kvq::g_encode_path.load(); }

kvq_status kvq_set_decode_path(int path) {
  if (path < 0 || path > 1) return fail(KVQ_ERR_INVALID_ARG, "set_decode_path: path must be 0 or 1");
  kvq::g_decode_path.store(path);
  return KVQ_OK;
}

int kvq_get_decode_path(void) { return kvq::g_decode_path.load(); }

kvq_status kvq_decode(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H, int T_cap,
                      int t0, int n, uint16_t* out, void* stream) {
  if (!p) return fail(KVQ_ERR_INVALID_ARG, "decode: null plan");
  if (B < 0 || H < 0 || n < 0 || T_cap < 0 || t0 < 0) return fail(KVQ_ERR_INVALID_ARG, "decode: negative size");
  if ((long)t0 + n > T_cap) return fail(KVQ_ERR_CAPACITY, "decode: t0 + n > T_cap");
  if (B == 0 || H == 0 || n == 0) return KVQ_OK;
  if (!out || !codes || !scales) return fail(KVQ_ERR_INVALID_ARG, "decode: null buffer");
  if (!kvq::aligned16(out) || !kvq::aligned16(codes) || !kvq::aligned16(scales))
    return fail(KVQ_ERR_ALIGNMENT, "decode: buffers must be 16-byte aligned");
  if ((long)B * H > (1L << 30) || (long)T_cap * B * H > (1L << 40)) return fail(KVQ_ERR_INVALID_ARG, "decode: too large");
  kvq_status st = kvq::check_plan_device(p);
  if (st != KVQ_OK) return st;
  if (kvq::decode_path() == 0)
    return kvq::launch_decode_tc(p, codes, scales, B, H, T_cap, t0, n, out, (cudaStream_t)stream);
  return kvq::launch_decode(p, codes, scales, B, H, T_cap, t0, n, out, (cudaStream_t)stream);
}

size_t kvq_workspace_size(int B, int Hq, int Hkv, int D, int T_cap) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T_cap < 0 || (D != 128 && D != 256) || Hq % Hkv) return 0;
  return kvq::attend_workspace_bytes(B, Hq, Hkv, D, T_cap);
}

static kvq_status check_attend_common(int B, int Hq, int Hkv, int D, int T_cap, int T_len, const void* q,
                                      const void* out, const void* ws, size_t ws_bytes) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T_cap < 0) return fail(KVQ_ERR_INVALID_ARG, "attend: bad sizes");
  if (Hq % Hkv) return fail(KVQ_ERR_UNSUPPORTED, "attend: Hq must be a multiple of Hkv");
  if (T_cap & 1) return fail(KVQ_ERR_ALIGNMENT, "attend: T_cap must be even");
  if (T_len < 0) return fail(KVQ_ERR_INVALID_ARG, "attend: T_len < 0");
  if (T_len > T_cap) return fail(KVQ_ERR_CAPACITY, "attend: T_len > T_cap");
  if (B == 0) return KVQ_OK;
  if (!q || !out) return fail(KVQ_ERR_INVALID_ARG, "attend: null buffer");
  if (!kvq::aligned16(q) || !kvq::aligned16(out)) return fail(KVQ_ERR_ALIGNMENT, "attend: q/out must be 16-byte aligned");
  const size_t need = kvq::attend_workspace_bytes(B, Hq, Hkv, D, T_cap);
  if (!ws || ws_bytes < need) return fail(KVQ_ERR_WORKSPACE, "attend: workspace missing or too small");
  if (!kvq::aligned16(ws)) return fail(KVQ_ERR_ALIGNMENT, "attend: workspace must be 16-byte aligned");
  return KVQ_OK;
}

kvq_status kvq_attend_decode(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                             const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq, int Hkv,
                             int T_cap, const int32_t* seq_lens, int T_len, float sigma, uint16_t* out,
                             void* ws, size_t ws_bytes, void* stream) {
  if (!pk || !pv) return fail(KVQ_ERR_INVALID_ARG, "attend: null plan");
  if (pk->D != pv->D || pk->G != pv->G || pk->device != pv->device || pk->xform != pv->xform ||
      pk->bits != pv->bits)
    return fail(KVQ_ERR_INVALID_ARG, "attend: K and V plans differ in head_dim, group, transform, code width or device");
  if (pk->G != 32 && pk->G != 16) return fail(KVQ_ERR_UNSUPPORTED, "attend: group must be 32 or 16");
  kvq_status st = check_attend_common(B, Hq, Hkv, pk->D, T_cap, T_len, q, out, ws, ws_bytes);
  if (st != KVQ_OK || B == 0) return st;
  if (!kc || !ks || !vc || !vs) return fail(KVQ_ERR_INVALID_ARG, "attend: null cache buffer");
  if (!kvq::aligned16(kc) || !kvq::aligned16(ks) || !kvq::aligned16(vc) || !kvq::aligned16(vs))
    return fail(KVQ_ERR_ALIGNMENT, "attend: cache buffers must be 16-byte aligned");
  st = kvq::check_plan_device(pk);
  if (st != KVQ_OK) return st;
  return kvq::launch_attend_int4(pk, pv, q, kc, ks, vc, vs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, out, ws,
                                 ws_bytes, (cudaStream_t)stream);
}

kvq_status kvq_attend_decode_append(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint16_t* k_new,
                                    const uint16_t* v_new, uint8_t* kc, uint16_t* ks, uint8_t* vc, uint16_t* vs, int B,
                                    int Hq, int Hkv, int T_cap, int pos, float sigma, uint16_t* out, void* ws,
                                    size_t ws_bytes, void* stream) {
  if (!pk || !pv) return fail(KVQ_ERR_INVALID_ARG, "attend_append: null plan");
  if (pk->D != pv->D || pk->G != pv->G || pk->device != pv->device || pk->xform != pv->xform ||
      pk->bits != pv->bits)
    return fail(KVQ_ERR_INVALID_ARG, "attend_append: K and V plans differ in head_dim, group, transform, code width or device");
  if (pk->G != 32 && pk->G != 16) return fail(KVQ_ERR_UNSUPPORTED, "attend_append: group must be 32 or 16");
  if (pos < 0) return fail(KVQ_ERR_INVALID_ARG, "attend_append: pos < 0");
  if (pos >= T_cap) return fail(KVQ_ERR_CAPACITY, "attend_append: pos + 1 > T_cap");
  kvq_status st = check_attend_common(B, Hq, Hkv, pk->D, T_cap, pos + 1, q, out, ws, ws_bytes);
  if (st != KVQ_OK || B == 0) return st;
  if (!kc || !ks || !vc || !vs) return fail(KVQ_ERR_INVALID_ARG, "attend_append: null cache buffer");
  if (!k_new || !v_new) return fail(KVQ_ERR_INVALID_ARG, "attend_append: null new K/V row");
  if (!kvq::aligned16(kc) || !kvq::aligned16(ks) || !kvq::aligned16(vc) || !kvq::aligned16(vs) ||
      !kvq::aligned16(k_new) || !kvq::aligned16(v_new))
    return fail(KVQ_ERR_ALIGNMENT, "attend_append: buffers must be 16-byte aligned");
  st = kvq::check_plan_device(pk);
  if (st != KVQ_OK) return st;
  return kvq::launch_attend_int4_append(pk, pv, q, k_new, v_new, kc, ks, vc, vs, B, Hq, Hkv, T_cap, pos, sigma, out,
                                        ws, ws_bytes, (cudaStream_t)stream);
}

kvq_status kvq_attend_decode_partial(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                                     const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq, int Hkv,
                                     int T_cap, int t_begin, int t_end, float sigma, float* partial, void* ws,
                                     size_t ws_bytes, void* stream) {
  if (!pk || !pv) return fail(KVQ_ERR_INVALID_ARG, "attend_partial: null plan");
  if (pk->D != pv->D || pk->G != pv->G || pk->device != pv->device || pk->xform != pv->xform ||
      pk->bits != pv->bits)
    return fail(KVQ_ERR_INVALID_ARG, "attend_partial: K and V plans differ in head_dim, group, transform, code width or device");
  if (pk->G != 32 && pk->G != 16) return fail(KVQ_ERR_UNSUPPORTED, "attend_partial: group must be 32 or 16");
  if (t_begin < 0 || t_end < t_begin) return fail(KVQ_ERR_INVALID_ARG, "attend_partial: need 0 <= t_begin <= t_end");
  if (t_end > T_cap) return fail(KVQ_ERR_CAPACITY, "attend_partial: t_end > T_cap");
  if (t_begin & 1) return fail(KVQ_ERR_ALIGNMENT, "attend_partial: t_begin must be even");
  kvq_status st = check_attend_common(B, Hq, Hkv, pk->D, T_cap, t_end - t_begin, q, partial, ws, ws_bytes);
  if (st != KVQ_OK || B == 0) return st;
  if (!kc || !ks || !vc || !vs) return fail(KVQ_ERR_INVALID_ARG, "attend_partial: null cache buffer");
  if (!kvq::aligned16(kc) || !kvq::aligned16(ks) || !kvq::aligned16(vc) || !kvq::aligned16(vs))
    return fail(KVQ_ERR_ALIGNMENT, "attend_partial: cache buffers must be 16-byte aligned");
  st = kvq::check_plan_device(pk);
  if (st != KVQ_OK) return st;
  return kvq::launch_attend_int4_partial(pk, pv, q, kc, ks, vc, vs, B, Hq, Hkv, T_cap, t_begin, t_end, sigma, partial,
                                         ws, ws_bytes, (cudaStream_t)stream);
}

kvq_status kvq_attend_combine(const kvq_plan* pv, const float* partials, int n_parts, int B, int Hq, uint16_t* out,
                              void* stream) {
  if (!pv) return fail(KVQ_ERR_INVALID_ARG, "attend_combine: null plan");
  if (n_parts < 1 || B < 0 || Hq <= 0) return fail(KVQ_ERR_INVALID_ARG, "attend_combine: bad sizes");
  if (B == 0) return KVQ_OK;
  if (!partials || !out) return fail(KVQ_ERR_INVALID_ARG, "attend_combine: null buffer");
  if (!kvq::aligned16(partials) || !kvq::aligned16(out))
    return fail(KVQ_ERR_ALIGNMENT, "attend_combine: buffers must be 16-byte aligned");
  kvq_status st = kvq::check_plan_device(pv);
  if (st != KVQ_OK) return st;
  return kvq::launch_attend_combine(pv, partials, n_parts, B, Hq, out, (cudaStream_t)stream);
}

kvq_status kvq_attend_decode_batch(const kvq_attend_job* jobs, int njobs, int B, int Hq, int Hkv, int T_cap,
                                   const int32_t* seq_lens, int T_len, float sigma, void* ws, size_t ws_bytes,
                                   void* stream) {
  if (njobs < 0 || (njobs > 0 && !jobs)) return fail(KVQ_ERR_INVALID_ARG, "attend_batch: bad job array");
  if (njobs == 0) return KVQ_OK;
  const kvq_plan* p0 = jobs[0].pk;
  if (!p0) return fail(KVQ_ERR_INVALID_ARG, "attend_batch: job 0: null plan");
  std::vector<kvq::AttendJobHost> hj((size_t)njobs);
  for (int i = 0; i < njobs; ++i) {
    const kvq_attend_job& j = jobs[i];
    const std::string tag = "attend_batch: job " + std::to_string(i) + ": ";
    if (!j.pk || !j.pv) return fail(KVQ_ERR_INVALID_ARG, tag + "null plan");
    if (j.pk->D != p0->D || j.pv->D != p0->D || j.pk->G != p0->G || j.pv->G != p0->G ||
        j.pk->device != p0->device || j.pv->device != p0->device || j.pk->xform != p0->xform ||
        j.pv->xform != p0->xform || j.pk->bits != p0->bits || j.pv->bits != p0->bits)
      return fail(KVQ_ERR_INVALID_ARG, tag + "plans differ in head_dim, group, transform, code width or device");
    if (j.pk->G != 32 && j.pk->G != 16) return fail(KVQ_ERR_UNSUPPORTED, tag + "group must be 32 or 16");
    kvq_status st = check_attend_common(B, Hq, Hkv, p0->D, T_cap, T_len, j.q, j.out, ws, ws_bytes);
    if (st != KVQ_OK) return fail(st, tag + kvq_last_error());
    if (B == 0) continue;
    if (!j.k_codes || !j.k_scales || !j.v_codes || !j.v_scales) return fail(KVQ_ERR_INVALID_ARG, tag + "null cache buffer");
    if (!kvq::aligned16(j.k_codes) || !kvq::aligned16(j.k_scales) || !kvq::aligned16(j.v_codes) ||
        !kvq::aligned16(j.v_scales))
      return fail(KVQ_ERR_ALIGNMENT, tag + "cache buffers must be 16-byte aligned");
    hj[(size_t)i] = kvq::AttendJobHost{j.pk, j.pv, j.q, j.k_codes, j.k_scales, j.v_codes, j.v_scales, j.out};
  }
  if (B == 0) return KVQ_OK;
  if ((size_t)B * std::min(njobs, 32) * Hkv > 65535u) return fail(KVQ_ERR_UNSUPPORTED, "attend_batch: 32 * B * Hkv > 65535");
  const size_t need = kvq::attend_workspace_bytes(B * std::min(njobs, 32), Hq, Hkv, p0->D, T_cap);
  if (ws_bytes < need) return fail(KVQ_ERR_WORKSPACE, "attend_batch: workspace too small (size it for min(njobs, 32) * B)");
  kvq_status st = kvq::check_plan_device(p0);
  if (st != KVQ_OK) return st;
  return kvq::launch_attend_int4_batch(hj.data(), njobs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, ws, ws_bytes,
                                       (cudaStream_t)stream);
}

kvq_status kvq_attend_decode_noalloc(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                                     const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq,
                                     int Hkv, int T_cap, const int32_t* seq_lens, int T_len, float sigma,
                                     uint16_t* out, void* stream) {
  if (!pk || !pv) return fail(KVQ_ERR_INVALID_ARG, "attend_noalloc: null plan");
  if (pk->D != pv->D || pk->G != pv->G || pk->device != pv->device || pk->xform != pv->xform ||
      pk->bits != pv->bits)
    return fail(KVQ_ERR_INVALID_ARG, "attend_noalloc: K and V plans differ in head_dim, group, transform, code width or device");
  if (pk->G != 32 && pk->G != 16) return fail(KVQ_ERR_UNSUPPORTED, "attend_noalloc: group must be 32 or 16");
  if (B < 0 || Hq <= 0 || Hkv <= 0 || T_cap < 0) return fail(KVQ_ERR_INVALID_ARG, "attend_noalloc: bad sizes");
  if (Hq % Hkv) return fail(KVQ_ERR_UNSUPPORTED, "attend_noalloc: Hq must be a multiple of Hkv");
  if (T_cap & 1) return fail(KVQ_ERR_ALIGNMENT, "attend_noalloc: T_cap must be even");
  if (T_len < 0) return fail(KVQ_ERR_INVALID_ARG, "attend_noalloc: T_len < 0");
  if (T_len > T_cap) return fail(KVQ_ERR_CAPACITY, "attend_noalloc: T_len > T_cap");
  if (B == 0) return KVQ_OK;
  if (!q || !out || !kc || !ks || !vc || !vs) return fail(KVQ_ERR_INVALID_ARG, "attend_noalloc: null buffer");
  if (!kvq::aligned16(q) || !kvq::aligned16(out) || !kvq::aligned16(kc) || !kvq::aligned16(ks) ||
      !kvq::aligned16(vc) || !kvq::aligned16(vs))
    return fail(KVQ_ERR_ALIGNMENT, "attend_noalloc: buffers must be 16-byte aligned");
  kvq_status st = kvq::check_plan_device(pk);
  if (st != KVQ_OK) return st;
  return kvq::launch_attend_int4_noalloc(pk, pv, q, kc, ks, vc, vs, B, Hq, Hkv, T_cap, seq_lens, T_len, sigma, out,
                                         (cudaStream_t)stream);
}

kvq_status kvq_attend_decode_ref(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq, int Hkv,
                                 int D, int T_cap, const int32_t* seq_lens, int T_len, float sigma, uint16_t* out,
                                 void* ws, size_t ws_bytes, void* stream) {
  if (D != 128 && D != 256) return fail(KVQ_ERR_UNSUPPORTED, "attend_ref: head_dim must be 128 or 256");
  kvq_status st = check_attend_common(B, Hq, Hkv, D, T_cap, T_len, q, out, ws, ws_bytes);
  if (st != KVQ_OK || B == 0) return st;
  if (!k || !v) return fail(KVQ_ERR_INVALID_ARG, "attend_ref: null cache buffer");
  if (!kvq::aligned16(k) || !kvq::aligned16(v)) return fail(KVQ_ERR_ALIGNMENT, "attend_ref: K/V must be 16-byte aligned");
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(KVQ_ERR_DEVICE, "attend_ref: no CUDA device");
  return kvq::launch_attend_fp16(q, k, v, B, Hq, Hkv, D, T_cap, seq_lens, T_len, sigma, out, ws, ws_bytes,
                                 (cudaStream_t)stream);
}

kvq_status kvq_attend_split_info(int B, int Hq, int Hkv, int D, int G, int bits, int T, int* splits, int* cluster,
                                 int* head_tiles) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || T < 0) return fail(KVQ_ERR_INVALID_ARG, "split_info: bad sizes");
  if (Hq % Hkv) return fail(KVQ_ERR_UNSUPPORTED, "split_info: Hq must be a multiple of Hkv");
  if (D != 128 && D != 256) return fail(KVQ_ERR_UNSUPPORTED, "split_info: head_dim must be 128 or 256");
  if (bits != 4 && bits != 8 && bits != 16) return fail(KVQ_ERR_UNSUPPORTED, "split_info: bits must be 4, 8 or 16");
  if (bits != 16 && G != 32 && G != 16) return fail(KVQ_ERR_UNSUPPORTED, "split_info: group must be 32 or 16");
  int dev = -1;
  cudaDeviceProp prop{};
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10)
    return fail(KVQ_ERR_DEVICE, "split_info: needs a current compute capability 10.x (sm_100) device");
  return kvq::attend_split_info(B, Hq, Hkv, D, G, bits, T, splits, cluster, head_tiles);
}

kvq_status kvq_debug_wait_timeout(uint32_t limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000u) return fail(KVQ_ERR_INVALID_ARG, "debug_wait_timeout: limit_us must be in [1, 1e6]");
  int dev = -1;
  cudaDeviceProp prop{};
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess || prop.major != 10)
    return fail(KVQ_ERR_DEVICE, "debug_wait_timeout: needs a current compute capability 10.x (sm_100) device");
  return kvq::launch_wait_probe(limit_us, (cudaStream_t)stream);
}

kvq_status kvq_poll_device_errors(uint32_t* flags) {
  if (cudaDeviceSynchronize() != cudaSuccess) return fail(KVQ_ERR_CUDA, "poll: device synchronize failed");
  const uint32_t f = kvq::codec_error_flags(true) | kvq::attend_error_flags(true) | kvq::encode_tc_error_flags(true) |
                     kvq::decode_tc_error_flags(true);
  if (flags) *flags = f;
  return KVQ_OK;
}

}  // extern "C"
