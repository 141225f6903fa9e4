// checks.cuh -- device bounds checks of the checked build.
//
// Compiled with -DMOE_DEBUG_CHECKS (libfp4moe_checked.so), every index a
// kernel takes from device data -- a routing target, an expert's entry in the
// location table, a padded row's token or pair -- is checked against the
// buffer it addresses before it is used.  A failed check records its code in
// the layer's error word (the first failure is kept; codes 201 and up, apart
// from the 1..99 of the bounded waits) and the access is skipped or redirected
// to an in-bounds element, so that a bad index surfaces as MOE_ERR_CUDA from
// the next moe_forward (this forward's outputs are invalid) instead of as a
// memory fault.  In the normal build every check is compiled out.
#pragma once

#include "moe_internal.h"
#include "tma.cuh"

namespace moe {

#ifdef MOE_DEBUG_CHECKS
constexpr bool kCheckedBuild = true;
#else
constexpr bool kCheckedBuild = false;
#endif

enum CheckCode {
  kChkTarget = 201,      // a routing target outside [0, targets)
  kChkLocExpert = 202,   // a location-table index outside [0, experts)
  kChkLocEntry = 203,    // a location outside the slot pool / staging ring
  kChkToken = 204,       // a padded row's token outside [-1, T) (or a real row's outside [0, T))
  kChkPair = 205,        // a padded row's pair outside [-1, T*k) (or a real row's outside [0, T*k))
};

// `ok`, recording `code` when it is false (checked build); true otherwise.
__device__ __forceinline__ bool dcheck(bool ok, int *err, int code) {
  if constexpr (kCheckedBuild) {
    if (!ok && err) record_first_error(err, code);
    return ok;
  } else {
    return true;
  }
}

// An index v read from device data, to lie in [lo, n): an index out of range
// is recorded and replaced by `safe`.
__device__ __forceinline__ int checked_index(int v, int lo, int n, int safe, int *err, int code) {
  return dcheck(v >= lo && v < n, err, code) ? v : safe;
}

// Where `expert`'s blob lives in this pass, from the location table; an
// expert index or an entry out of range reads as absent (checked build).
__device__ __forceinline__ int load_loc(const int *table, int expert, const DevBounds &b) {
  if (!dcheck(expert >= 0 && expert < b.n_experts, b.err, kChkLocExpert)) return kLocAbsent;
  const int loc = __ldcg(table + expert);
  const bool ok = loc == kLocAbsent || (loc >= 0 ? loc < b.n_slots : (-2 - loc) < b.n_staging);
  return dcheck(ok, b.err, kChkLocEntry) ? loc : kLocAbsent;
}

}  // namespace moe
