// pa_calib.cu -- per-SM shares of the decode kernel's work, measured once.
//
// The decode kernel is bound by HBM and hands every warp a fixed contiguous
// range of the batch's key tiles before it starts (no claims at run time, so
// the result does not depend on timing).  On a B200 the SMs do not stream
// equally fast under a full load: timed per warp, pairs of SMs move about 44,
// 51 or 59 GB/s, the same pattern from launch to launch.  With equal shares
// the GPU then idles while its slowest SMs finish.  pa_calibrate runs the
// decode kernel itself on a synthetic batch, times every SM's share with the
// global timer, and adjusts per-SM weights until the SMs finish together;
// later decode launches copy the weights into their parameters and give each
// SM a share in proportion to its weight.  The split stays a pure function of
// the batch and of the recorded weights.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include "pa_internal.h"

namespace pa {

namespace {

// The synthetic batch: 128 sequences of 2048 tokens, 64 query / 8 KV heads,
// head_dim 128, 16-token blocks (the 70B-like decode layer's shape), blocks
// taken from the pool in a shuffled order.
constexpr int CAL_SEQS = 128, CAL_CTX = 2048, CAL_HQ = 64, CAL_HKV = 8, CAL_D = 128, CAL_BS = 16;
constexpr int CAL_BLOCKS_PER_SEQ = CAL_CTX / CAL_BS;
constexpr int CAL_NB = CAL_SEQS * CAL_BLOCKS_PER_SEQ;
constexpr size_t CAL_CACHE_BYTES = static_cast<size_t>(CAL_NB) * CAL_HKV * CAL_BS * CAL_D * 2;
constexpr int CAL_ROUNDS = 4;    // 1 with equal shares, then 3 corrections
constexpr int CAL_LAUNCHES = 2;  // timed launches per round (their times are averaged)

size_t al256(size_t n) { return (n + 255) / 256 * 256; }

struct DeviceRates {
  bool valid;
  int num_sms;
  uint16_t rate[PA_MAX_WEIGHTED_SMS];
};

std::mutex g_rates_mu;
DeviceRates g_rates[PA_MAX_DEVICES] = {};

// The bytes pa_calibrate needs in its buffer on the current device.
size_t calib_bytes(int num_sms, size_t* ws_bytes) {
  const size_t ws = decode_workspace_bytes(CAL_SEQS, CAL_HQ, CAL_HKV, CAL_D, CAL_BLOCKS_PER_SEQ, CAL_BS);
  if (ws_bytes) *ws_bytes = ws;
  const size_t small = al256(CAL_SEQS * CAL_BLOCKS_PER_SEQ * 4) + al256(CAL_SEQS * 4) +
                       2 * al256(static_cast<size_t>(CAL_SEQS) * CAL_HQ * CAL_D * 2) +
                       al256(static_cast<size_t>(num_sms) * 3 * 4 * 4 * 8);  // trace: 4 words per warp
  return 2 * CAL_CACHE_BYTES + small + al256(ws);
}

}  // namespace

bool sm_rates_snapshot(uint16_t* out, int num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= PA_MAX_DEVICES) return false;
  std::lock_guard<std::mutex> lock(g_rates_mu);
  const DeviceRates& r = g_rates[dev];
  if (!r.valid || r.num_sms != num_sms) return false;
  for (int i = 0; i < num_sms; ++i) out[i] = r.rate[i];
  return true;
}

void sm_rates_clear() {
  std::lock_guard<std::mutex> lock(g_rates_mu);
  for (auto& r : g_rates) r.valid = false;
}

}  // namespace pa

extern "C" size_t pa_calibrate_bytes(void) {
  pa::DeviceInfo di;
  if (pa::device_info(&di) != PA_OK) return 0;
  return pa::calib_bytes(di.num_sms, nullptr);
}

extern "C" int pa_calibrate(void* buffer, size_t bytes, int* dev_status, void* stream) {
  using namespace pa;
  if (!buffer) return PA_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(buffer) & 255) != 0) return PA_ERR_SHAPE;
  DeviceInfo di;
  int rc = device_info(&di);
  if (rc != PA_OK) return rc;
  if (di.num_sms > PA_MAX_WEIGHTED_SMS) return PA_ERR_UNSUPPORTED;
  size_t ws_bytes = 0;
  if (bytes < calib_bytes(di.num_sms, &ws_bytes) || ws_bytes == 0) return PA_ERR_WORKSPACE;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  const cudaStream_t st = static_cast<cudaStream_t>(stream);

  // carve the buffer: K cache, V cache, tables, lengths, q, out, trace, workspace
  uint8_t* b = static_cast<uint8_t*>(buffer);
  void* kc = b;
  b += CAL_CACHE_BYTES;
  void* vc = b;
  b += CAL_CACHE_BYTES;
  int32_t* tables = reinterpret_cast<int32_t*>(b);
  b += al256(CAL_SEQS * CAL_BLOCKS_PER_SEQ * 4);
  int32_t* ctx = reinterpret_cast<int32_t*>(b);
  b += al256(CAL_SEQS * 4);
  void* q = b;
  b += al256(static_cast<size_t>(CAL_SEQS) * CAL_HQ * CAL_D * 2);
  void* out = b;
  b += al256(static_cast<size_t>(CAL_SEQS) * CAL_HQ * CAL_D * 2);
  const size_t trace_words = static_cast<size_t>(di.num_sms) * 3 * 4 * 4;
  unsigned long long* trace = reinterpret_cast<unsigned long long*>(b);
  b += al256(trace_words * 8);
  void* ws = b;

  // the batch, made on the host: a fixed shuffle of the pool (a 64-bit LCG)
  std::vector<int32_t> h_tables(CAL_NB), h_ctx(CAL_SEQS, CAL_CTX);
  for (int i = 0; i < CAL_NB; ++i) h_tables[i] = i;
  uint64_t x = 0x9e3779b97f4a7c15ull;
  for (int i = CAL_NB - 1; i > 0; --i) {
    x = x * 6364136223846793005ull + 1442695040888963407ull;
    const int j = static_cast<int>((x >> 33) % static_cast<uint64_t>(i + 1));
    std::swap(h_tables[i], h_tables[j]);
  }
  if ((e = cudaMemcpyAsync(tables, h_tables.data(), CAL_NB * 4, cudaMemcpyHostToDevice, st)) != cudaSuccess ||
      (e = cudaMemcpyAsync(ctx, h_ctx.data(), CAL_SEQS * 4, cudaMemcpyHostToDevice, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(q, 0, static_cast<size_t>(CAL_SEQS) * CAL_HQ * CAL_D * 2, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(ws, 0, ws_bytes, st)) != cudaSuccess)
    return cuda_fail(e, "calibration set-up copy");

  const int S = di.num_sms;
  std::vector<double> weight(S, 1.0), time_s(S), bytes_s(S);
  std::vector<unsigned long long> h_trace(trace_words);
  std::vector<uint16_t> w16(S, 1);
  for (int round = 0; round < CAL_ROUNDS; ++round) {
    // weights as the launch carries them (uint16, largest 60000)
    const double wmax = *std::max_element(weight.begin(), weight.end());
    for (int i = 0; i < S; ++i) w16[i] = static_cast<uint16_t>(std::max(1.0, std::round(weight[i] / wmax * 60000.0)));
    RowsOverride ovr{trace, round == 0 ? 0 : 1, w16.data()};
    std::fill(time_s.begin(), time_s.end(), 0.0);
    std::fill(bytes_s.begin(), bytes_s.end(), 0.0);
    for (int l = 0; l < CAL_LAUNCHES + 1; ++l) {  // the first launch of a round is not timed
      if ((e = cudaMemsetAsync(trace, 0, trace_words * 8, st)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
      rc = run_attention(out, q, nullptr, kc, vc, tables, CAL_BLOCKS_PER_SEQ, ctx, CAL_SEQS, CAL_SEQS, CAL_HQ, CAL_HKV,
                         CAL_D, CAL_BS, CAL_NB, 0.088f, ws, ws_bytes, dev_status, stream, nullptr, nullptr, nullptr,
                         nullptr, 0, 0, 1.f, 1.f, nullptr, &ovr);
      if (rc != PA_OK) return rc;
      if (l == 0) continue;
      if ((e = cudaMemcpyAsync(h_trace.data(), trace, trace_words * 8, cudaMemcpyDeviceToHost, st)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpyAsync");
      if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
      // per SM: its bytes over the time from its first copy to its last tile
      std::vector<unsigned long long> t0(S, ~0ull), t1(S, 0);
      std::vector<double> by(S, 0.0);
      for (size_t r = 0; r + 3 < trace_words; r += 4) {
        const unsigned long long sm = h_trace[r], units = h_trace[r + 1], a = h_trace[r + 2], z = h_trace[r + 3];
        if (z == 0 || units == 0 || sm >= static_cast<unsigned long long>(S)) continue;
        t0[sm] = std::min(t0[sm], a);
        t1[sm] = std::max(t1[sm], z);
        by[sm] += static_cast<double>(units) * CAL_BS * CAL_D * 4;  // K and V of 16 keys
      }
      for (int i = 0; i < S; ++i) {
        if (t1[i] <= t0[i] || t0[i] == ~0ull) return PA_ERR_RANGE;  // an SM without work: keep the equal split
        time_s[i] += static_cast<double>(t1[i] - t0[i]) / CAL_LAUNCHES;
        bytes_s[i] += by[i] / CAL_LAUNCHES;
      }
    }
    if (round == 0) {  // shares in proportion to the rates seen with equal shares
      for (int i = 0; i < S; ++i) weight[i] = bytes_s[i] / time_s[i];
    } else {  // move every SM's share towards the mean finishing time
      double mean = 0.0;
      for (int i = 0; i < S; ++i) mean += time_s[i] / S;
      for (int i = 0; i < S; ++i) weight[i] *= std::pow(mean / time_s[i], 0.7);
    }
  }
  DeviceRates r{};
  r.valid = true;
  r.num_sms = S;
  const double wmax = *std::max_element(weight.begin(), weight.end());
  for (int i = 0; i < S; ++i) r.rate[i] = static_cast<uint16_t>(std::max(1.0, std::round(weight[i] / wmax * 60000.0)));
  std::lock_guard<std::mutex> lock(g_rates_mu);
  g_rates[dev] = r;
  return PA_OK;
}

extern "C" int pa_calibration(int* num_sms, uint16_t* weights_out) {
  if (!num_sms) return PA_ERR_NULL;
  pa::DeviceInfo di;
  int rc = pa::device_info(&di);
  if (rc != PA_OK) return rc;
  *num_sms = di.num_sms;
  uint16_t tmp[pa::PA_MAX_WEIGHTED_SMS];
  if (di.num_sms > pa::PA_MAX_WEIGHTED_SMS || !pa::sm_rates_snapshot(tmp, di.num_sms)) return PA_ERR_RANGE;
  if (weights_out)
    for (int i = 0; i < di.num_sms; ++i) weights_out[i] = tmp[i];
  return PA_OK;
}

extern "C" void pa_calibration_clear(void) { pa::sm_rates_clear(); }
