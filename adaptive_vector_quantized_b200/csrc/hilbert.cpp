// Host-side Hilbert curve over a 2^k x 2^k grid: the power-of-two case of the
// generalised Hilbert ("Gilbert") token order of "AVQ-Attention: Adaptive
// Vector-Quantized Attention", Sec. 4.2 and Fig. 3.  Quadrant-rotation
// construction: at each scale the two index bits pick a quadrant, and the
// lower-scale coordinates are reflected or transposed so that the curve stays
// continuous.
#include <stdint.h>

#include "avq.h"

namespace {

void hilbert_cell(int side, int64_t t, int* x_out, int* y_out) {
  int x = 0, y = 0;
  for (int s = 1; s < side; s *= 2) {
    const int rx = (int)((t / 2) & 1);
    const int ry = (int)((t ^ rx) & 1);
    if (ry == 0) {
      if (rx == 1) {
        x = s - 1 - x;
        y = s - 1 - y;
      }
      const int tmp = x;
      x = y;
      y = tmp;
    }
    x += s * rx;
    y += s * ry;
    t /= 4;
  }
  *x_out = x;
  *y_out = y;
}

}  // namespace

extern "C" avq_status avq_hilbert_order(int side, int32_t* idx) {
  if (side < 1 || (side & (side - 1)) != 0 || side > 32768 || idx == nullptr)
    return AVQ_ERR_INVALID_ARG;
  const int64_t n = (int64_t)side * side;
  for (int64_t t = 0; t < n; ++t) {
    int x, y;
    hilbert_cell(side, t, &x, &y);
    idx[t] = (int32_t)((int64_t)y * side + x);
  }
  return AVQ_OK;
}
