// Measured policy map and the dispatcher built on it.
//
// ADAngel page (awesome-system-papers, OSDI'26, core method): an offline script runs every
// candidate kernel of the strategy set over the (M, N, K) and bit-width combinations a
// model will meet, times each with CUDA events, keeps the fastest as the "oracle policy
// map", and the runtime dispatcher only looks the shape and bit width up in that table
// before calling the chosen kernel.  Here the strategy set is the fused GEMV (with its
// warps-per-unit and grid-size variants; over 16-row slices of x when M > 16) and the
// prefill path (stand-alone dequantization + dense GEMM); the offline script is the
// package's tune module.  The table lives in host memory, is installed whole by
// qlinear_policy_set and read under a mutex on every planned call.
#include <climits>
#include <mutex>
#include <vector>

#include "policy.h"
#include "qlinear.h"

namespace {

std::mutex g_mu;
std::vector<ql_policy_entry> g_table;

bool fmt_ok(int fmt) { return fmt == 2 || fmt == 4 || fmt == 8 || fmt == 16; }

// Built-in rule (no table entry): the GEMV while its per-16-row cost stays below a
// dequantization plus a GEMM (measured crossover between M = 64 and M = 96 on the
// 8192 x 28672 layer), prefill above.
constexpr int kRulePrefillAbove = 64;

}  // namespace

namespace qpolicy {

Choice lookup(int fmt, bool outl, int M, int N, int K) {
  if (!outl) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (const ql_policy_entry& e : g_table)
      if (e.fmt == fmt && e.N == N && e.K == K && M >= e.m_lo && M <= e.m_hi)
        return Choice{e.strategy, e.warps_per_unit, e.ctas, true};
  }
  return Choice{M > kRulePrefillAbove && !outl ? QL_STRATEGY_PREFILL : QL_STRATEGY_GEMV, 0, 0,
                false};
}

}  // namespace qpolicy

extern "C" ql_status qlinear_policy_set(const ql_policy_entry* entries, int n) {
  if (n < 0) return QL_ERR_SHAPE;
  if (n > 0 && !entries) return QL_ERR_NULL;
  for (int i = 0; i < n; ++i) {
    const ql_policy_entry& e = entries[i];
    if (!fmt_ok(e.fmt)) return QL_ERR_UNSUPPORTED;
    if (e.strategy != QL_STRATEGY_GEMV && e.strategy != QL_STRATEGY_PREFILL)
      return QL_ERR_UNSUPPORTED;
    if (e.N <= 0 || e.K <= 0 || e.N % 16 || e.K % 128 || e.m_lo < 1 || e.m_hi < e.m_lo)
      return QL_ERR_SHAPE;
    if (e.warps_per_unit != 0 && e.warps_per_unit != 1 && e.warps_per_unit != 2 &&
        e.warps_per_unit != 4)
      return QL_ERR_SHAPE;
    if (e.ctas < 0) return QL_ERR_SHAPE;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  g_table.assign(entries, entries + n);
  return QL_OK;
}

extern "C" int qlinear_policy_size(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  return (int)g_table.size();
}

extern "C" ql_status qlinear_policy_lookup(int fmt, int M, int N, int K, ql_policy_entry* out,
                                           int* from_table) {
  if (!out) return QL_ERR_NULL;
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (M < 1 || N <= 0 || K <= 0) return QL_ERR_SHAPE;
  const qpolicy::Choice c = qpolicy::lookup(fmt, false, M, N, K);
  ql_policy_entry r{fmt, N, K, M, M, c.strategy, c.wpu, c.ctas};
  if (c.from_table) {
    std::lock_guard<std::mutex> lk(g_mu);
    for (const ql_policy_entry& e : g_table)
      if (e.fmt == fmt && e.N == N && e.K == K && M >= e.m_lo && M <= e.m_hi) {
        r = e;
        break;
      }
  } else if (M > kRulePrefillAbove) {
    r.m_lo = kRulePrefillAbove + 1;
    r.m_hi = INT_MAX;
  } else {
    r.m_lo = 1;
    r.m_hi = kRulePrefillAbove;
  }
  *out = r;
  if (from_table) *from_table = c.from_table ? 1 : 0;
  return QL_OK;
}

extern "C" ql_status qlinear_matmul(int fmt, const uint16_t* x, const void* packed,
                                    const void* p0, const void* p1, uint16_t* y, int M, int N,
                                    int K, void* workspace, size_t workspace_bytes,
                                    uint16_t* w_fp16, ql_stream_t stream) {
  if (!fmt_ok(fmt)) return QL_ERR_UNSUPPORTED;
  if (M < 1) return QL_ERR_SHAPE;
  const qpolicy::Choice c = qpolicy::lookup(fmt, false, M, N, K);
  if (c.strategy == QL_STRATEGY_PREFILL) {
    if (w_fp16) return qlinear_prefill(fmt, x, packed, p0, p1, w_fp16, y, M, N, K, stream);
    // the tensor-core GEMM with the dequantization fused in, whole tiles per CTA (the GEMV
    // workspace is not the stream-K workspace)
    return qlinear_prefill_fused(fmt, x, packed, p0, p1, y, M, N, K, nullptr, 0, stream);
  }
  // the fused GEMV, over 16-row slices of x and y
  if (!x || !y) return QL_ERR_NULL;
  for (int m0 = 0; m0 < M; m0 += 16) {
    const int m = M - m0 < 16 ? M - m0 : 16;
    const uint16_t* xs = x + (size_t)m0 * K;
    uint16_t* ys = y + (size_t)m0 * N;
    ql_status st;
    switch (fmt) {
      case QL_FMT_W2:
        st = qlinear_w2a16(xs, static_cast<const uint32_t*>(packed),
                           static_cast<const uint16_t*>(p0), static_cast<const uint16_t*>(p1), ys,
                           m, N, K, 128, workspace, workspace_bytes, stream);
        break;
      case QL_FMT_W4:
        st = qlinear_w4a16(xs, static_cast<const uint32_t*>(packed),
                           static_cast<const uint16_t*>(p0), static_cast<const uint16_t*>(p1), ys,
                           m, N, K, 128, workspace, workspace_bytes, stream);
        break;
      case QL_FMT_W8:
        st = qlinear_w8a16(xs, static_cast<const uint32_t*>(packed),
                           static_cast<const uint16_t*>(p0), static_cast<const uint16_t*>(p1), ys,
                           m, N, K, 128, workspace, workspace_bytes, stream);
        break;
      default:
        st = qlinear_lut4(xs, static_cast<const uint8_t*>(packed),
                          static_cast<const uint16_t*>(p0), static_cast<const float*>(p1), ys, m,
                          N, K, 64, workspace, workspace_bytes, stream);
        break;
    }
    if (st != QL_OK) return st;
  }
  return QL_OK;
}
