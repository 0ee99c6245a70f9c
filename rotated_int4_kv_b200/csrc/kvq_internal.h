// kvq_internal.h -- definitions shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <string>
#include <type_traits>

#include "../../include/kvq.h"

namespace kvq {

constexpr int kMaxD = 256;

// Per-plan constants handed to the codec kernels by value (kernel parameter
// space), so that every per-channel factor is a constant-bank operand.
struct CodecConsts {
  float chan[kMaxD];       // encode: lambda_c * dg_c ; decode: dg_c / lambda_c (rotated channel c)
  uint32_t sgn[kMaxD / 2]; // XOR mask per fp16 pair of the original domain (0x8000 per negative s)
};

}  // namespace kvq

struct kvq_plan {
  int D = 0;
  int G = 0;
  int device = -1;
  int xform = 0;           // kvq_transform: 0 SRFT, 1 SRHT
  int bits = 4;            // code width: 4 (nibble pairs) or 8 (one byte per channel)
  kvq::CodecConsts enc{};  // lambda_c * dg_c
  kvq::CodecConsts dec{};  // dg_c / lambda_c
  // Device block: copies of `enc` and `dec` for kernels that serve several plans
  // in one launch (grouped encode) or two plans at once (attention: K and V).
  void* dblock = nullptr;
  const kvq::CodecConsts* enc_dev = nullptr;
  const kvq::CodecConsts* dec_dev = nullptr;
  // Tensor-core encode operand in the same block: W = Lambda F_r diag(s) as fp16
  // hi + lo, per 128-channel half 128 hi rows then 128 lo rows, D columns.
  const uint16_t* wt_dev = nullptr;
  // Attention operand in the same block: F128, the unnormalised 128-point real DFT in
  // slot order, fp16 hi rows [128] then lo rows [128] (plan-independent; the attention
  // kernels apply the plans' signs and per-channel factors around it).
  const uint16_t* rot_dev = nullptr;
  // Tensor-core decode operand in the same block: W_dec = diag(s) Q^T Lambda^-1 as fp16,
  // D rows (output samples) x D columns (channels, in the dequantiser's pair order).
  const uint16_t* wdec_dev = nullptr;
};

namespace kvq {

// Bytes of one cached vector's codes.
inline int code_row_bytes(const kvq_plan* p) { return p->D * p->bits / 8; }

template <int V>
using IC = std::integral_constant<int, V>;

// Calls f(IC<D>, IC<G>, IC<BITS>) for the quantiser configurations the kernels are
// built for (D 128 | 256, G 32 | 16, BITS 4 | 8); fails with `what` otherwise.
template <typename F>
auto dispatch_dgb(int D, int G, int bits, F&& f) -> decltype(f(IC<128>{}, IC<32>{}, IC<4>{})) {
  if (bits == 4) {
    if (D == 128) return G == 32 ? f(IC<128>{}, IC<32>{}, IC<4>{}) : f(IC<128>{}, IC<16>{}, IC<4>{});
    return G == 32 ? f(IC<256>{}, IC<32>{}, IC<4>{}) : f(IC<256>{}, IC<16>{}, IC<4>{});
  }
  if (D == 128) return G == 32 ? f(IC<128>{}, IC<32>{}, IC<8>{}) : f(IC<128>{}, IC<16>{}, IC<8>{});
  return G == 32 ? f(IC<256>{}, IC<32>{}, IC<8>{}) : f(IC<256>{}, IC<16>{}, IC<8>{});
}

// thread-local last-error text
void set_error(const std::string& msg);
kvq_status fail(kvq_status st, const std::string& msg);

// driver entry point for tensor-map encoding (no link against libcuda)
kvq_status encode_tiled(CUtensorMap* map, CUtensorMapDataType dt, int rank, const void* base,
                        const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                        CUtensorMapSwizzle swz, const char* what);

int num_sms(int device);

kvq_status check_plan_device(const kvq_plan* p);

// tensor-core encode (kvq_encode_tc.cu)
bool encode_tc_supported(int D, int G);
bool encode_split_supported(const kvq_plan* p);
kvq_status launch_encode_tc(const kvq_encode_job* jobs, int njobs, cudaStream_t s, bool split);
uint32_t encode_tc_error_flags(bool clear);
// encode path: 0 = tensor cores where supported (the radix-2 split kernel for head_dim 256 SRFT
// plans), else the register FFT; 1 = register FFT; 2 = tensor cores, dense product; 3 = tensor
// cores, radix-2 split (head_dim 256 SRFT only)
int encode_path();
kvq_status dispatch_encode(const kvq_encode_job* jobs, int njobs, cudaStream_t s);

// tensor-core decode (kvq_decode_tc.cu)
kvq_status launch_decode_tc(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H,
                            int T_cap, int t0, int n, uint16_t* out, cudaStream_t s);
uint32_t decode_tc_error_flags(bool clear);
// decode path: 0 = tensor cores (default), 1 = register FFT
int decode_path();
// K position p (0..7) of a 16-byte unit of the tensor-core decode's fp16 operand -> the
// channel offset within the unit's eight channels (the dequantiser's pair order)
inline int decode_unit_channel(int p, int bits) {
  if (bits == 4) return (p & 1) ? (p >> 1) + 4 : (p >> 1);  // pairs (j, j + 4) of one 32-bit word
  static const int k8[8] = {0, 2, 1, 3, 4, 6, 5, 7};       // pairs (0, 2), (1, 3) of each word
  return k8[p];
}

// codec launchers (kvq_codec.cu)
kvq_status launch_encode_jobs(const kvq_encode_job* jobs, int njobs, cudaStream_t s);
kvq_status launch_decode(const kvq_plan* p, const uint8_t* codes, const uint16_t* scales, int B, int H,
                         int T_cap, int t0, int n, uint16_t* out, cudaStream_t s);

// attention launchers (kvq_attend.cu)
// One decode-attention problem: plans (quantised caches; none for the fp16 comparator),
// query, caches, output.
struct AttendJobHost {
  const kvq_plan* pk;
  const kvq_plan* pv;
  const uint16_t* q;
  const void* kc;   // K codes (int4) or fp16 K
  const uint16_t* ks;
  const void* vc;   // V codes (int4) or fp16 V
  const uint16_t* vs;
  uint16_t* out;
};
size_t attend_workspace_bytes(int B, int Hq, int Hkv, int D, int T_cap);
kvq_status launch_attend_int4_batch(const AttendJobHost* jobs, int njobs, int B, int Hq, int Hkv, int T_cap,
                                    const int32_t* seq_lens, int T_len, float sigma, void* ws, size_t ws_bytes,
                                    cudaStream_t s);
kvq_status launch_attend_int4(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q,
                              const uint8_t* kc, const uint16_t* ks, const uint8_t* vc, const uint16_t* vs,
                              int B, int Hq, int Hkv, int T_cap, const int32_t* seq_lens, int T_len,
                              float sigma, uint16_t* out, void* ws, size_t ws_bytes, cudaStream_t s);
kvq_status launch_attend_int4_noalloc(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q,
                                      const uint8_t* kc, const uint16_t* ks, const uint8_t* vc,
                                      const uint16_t* vs, int B, int Hq, int Hkv, int T_cap,
                                      const int32_t* seq_lens, int T_len, float sigma, uint16_t* out,
                                      cudaStream_t s);
kvq_status launch_attend_int4_append(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint16_t* k_new,
                                     const uint16_t* v_new, uint8_t* kc, uint16_t* ks, uint8_t* vc, uint16_t* vs, int B,
                                     int Hq, int Hkv, int T_cap, int pos, float sigma, uint16_t* out, void* ws,
                                     size_t ws_bytes, cudaStream_t s);
kvq_status launch_attend_int4_partial(const kvq_plan* pk, const kvq_plan* pv, const uint16_t* q, const uint8_t* kc,
                                      const uint16_t* ks, const uint8_t* vc, const uint16_t* vs, int B, int Hq,
                                      int Hkv, int T_cap, int t_begin, int t_end, float sigma, float* part, void* ws,
                                      size_t ws_bytes, cudaStream_t s);
kvq_status launch_attend_combine(const kvq_plan* pv, const float* parts, int N, int B, int Hq, uint16_t* out,
                                 cudaStream_t s);
kvq_status launch_attend_fp16(const uint16_t* q, const uint16_t* k, const uint16_t* v, int B, int Hq,
                              int Hkv, int D, int T_cap, const int32_t* seq_lens, int T_len, float sigma,
                              uint16_t* out, void* ws, size_t ws_bytes, cudaStream_t s);

kvq_status attend_split_info(int B, int Hq, int Hkv, int D, int G, int bits, int T, int* splits, int* cluster,
                             int* head_tiles);
kvq_status launch_wait_probe(uint32_t limit_us, cudaStream_t s);

// device error word (bit flags raised by kernels that gave up a bounded wait)
uint32_t* device_error_word();

}  // namespace kvq
