// Measured policy map: the host-side table that picks, per (format, N, K, M), the strategy
// and GEMV launch variant.  Internal interface between the table (policy.cpp) and the GEMV
// planner (qlinear.cu).
#pragma once

namespace qpolicy {

struct Choice {
  int strategy;  // QL_STRATEGY_GEMV or QL_STRATEGY_PREFILL
  int wpu;       // 0 = planner's rule, else warps per unit
  int ctas;      // 0 = planner's rule, else grid size
  bool from_table;
};

// The table entry covering (fmt, M, N, K), else the built-in rule.  Outlier layers are not
// in the table (the rule applies).
Choice lookup(int fmt, bool outl, int M, int N, int K);

}  // namespace qpolicy
