// A flattened index v = i * per_row + j over the rows of a matrix, walked in fixed strides by
// the elementwise passes: one division when a thread starts, then an add and at most one wrap
// per step (a 64-bit division per 16-byte vector cost as many instructions as the pass's own
// arithmetic).
#pragma once

namespace muon {

struct RowPos {
  int i, j;  // row, position within the row
};

// The position of flattened index v (one division).
__device__ __forceinline__ RowPos rowpos_at(long long v, int per_row) {
  const long long i = v / per_row;
  return RowPos{static_cast<int>(i), static_cast<int>(v - i * per_row)};
}

// A stride split once into whole rows and a remainder (< per_row).
struct RowStep {
  int rows, rem;
};

__device__ __forceinline__ RowStep rowstep_of(int stride, int per_row) {
  return RowStep{stride / per_row, stride % per_row};
}

__device__ __forceinline__ RowPos rowpos_add(RowPos p, RowStep s, int per_row) {
  p.i += s.rows;
  p.j += s.rem;
  if (p.j >= per_row) {
    p.j -= per_row;
    ++p.i;
  }
  return p;
}

}  // namespace muon
