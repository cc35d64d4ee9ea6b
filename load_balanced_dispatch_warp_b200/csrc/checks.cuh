// Host-side argument rules of the C ABI, shared by every entry point that takes the same
// sizes (one copy of each rule, so two entry points over the same operation cannot drift
// apart).  Each returns MOE_OK or the status the header documents.
#pragma once

#include <stdint.h>

#include "moe.h"

namespace moe {
namespace checks {

constexpr int64_t kMaxElems = (int64_t)1 << 31;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 1 <= k <= min(E, 32), E <= 1024, T >= 0, T*E and T*k below 2^31.
inline int route(int T, int E, int k) {
  if (T < 0 || E < 1 || k < 1) return MOE_ERR_ARG;
  if (E > 1024 || k > E || k > 32) return MOE_ERR_SHAPE;
  if ((int64_t)T * E >= kMaxElems || (int64_t)T * k >= kMaxElems) return MOE_ERR_SHAPE;
  return MOE_OK;
}

// E % R == 0, R <= E, and (when rows are laid out per rank) T*k % R == 0.
inline int ranks(int T, int k, int E, int R, bool need_even_rows) {
  if (R < 1) return MOE_ERR_ARG;
  if (R > E || E % R != 0) return MOE_ERR_SHAPE;
  if (need_even_rows && ((int64_t)T * k) % R != 0) return MOE_ERR_SHAPE;
  return MOE_OK;
}

// d % 128 == 0, F % 128 == 0, and every [rows, d], [rows, F], [T, d] tensor below 2^31.
inline int dims(int T, int k, int d, int F) {
  if (d < 1 || F < 1) return MOE_ERR_ARG;
  if (d % 128 != 0 || F % 128 != 0) return MOE_ERR_SHAPE;
  const int64_t rows = (int64_t)T * k;
  if (rows * d >= kMaxElems || rows * F >= kMaxElems || (int64_t)T * d >= kMaxElems)
    return MOE_ERR_SHAPE;
  return MOE_OK;
}

// S >= 0 and at most 4096 groups in the plan (R * (E/R + S)).
inline int groups(int E, int R, int S) {
  if (S < 0) return MOE_ERR_ARG;
  if ((int64_t)R * (E / R + S) > 4096) return MOE_ERR_SHAPE;
  return MOE_OK;
}

// The rules of moe_dispatch (and of every call with its arguments): pointers, sizes and
// 16-byte alignment of the row tensors.  `workspace` is checked by the caller.
inline int dispatch(const void* x, const int32_t* idx, const int32_t* plan, int T, int k, int E,
                    int R, int S, int d, const void* recv, const int32_t* perm,
                    const int32_t* src, const int32_t* err) {
  if (!plan || !err) return MOE_ERR_ARG;
  if (T > 0 && (!x || !idx || !recv || !perm || !src)) return MOE_ERR_ARG;
  int st = route(T, E, k);
  if (st == MOE_OK) st = ranks(T, k, E, R, true);
  if (st == MOE_OK) st = groups(E, R, S);
  if (st == MOE_OK) st = dims(T, k, d, 128);
  if (st != MOE_OK) return st;
  if (!aligned16(x) || !aligned16(recv)) return MOE_ERR_ARG;
  return MOE_OK;
}

}  // namespace checks
}  // namespace moe
