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

// ---------------------------------------------------------------------------
// Generalised Hilbert order over a width x height grid of any size (the
// "Gilbert" order of Sec. 4.2 and Fig. 3, e.g. the 28 x 28 patch grid).
//
// The curve is built as a Hamiltonian path of the grid graph between two
// corners of one side, by recursive splitting.  A block is given by a corner,
// a travel direction along which its path goes from that corner to the next
// corner (la cells) and a side direction (lb cells).  Colouring the cells like
// a chessboard, such a path exists exactly when la is even or both la and lb
// are odd, and every split below keeps that property for its parts:
//   - lb == 1: a straight line; la == 2: up the side direction and back;
//   - a long block (la >= 2 lb, or lb == 2): two halves along the travel
//     direction, the split point even when lb is even;
//   - otherwise the Hilbert "U": the first a = la/2 columns of the near strip
//     (b rows, b even) walked along the side direction, the far strip of
//     lb - b rows walked along the travel direction, the last la - a columns
//     of the near strip walked back to the far corner.
// On a 2^k x 2^k grid every split is the Hilbert quadrant split, so the
// order equals avq_hilbert_order's.
namespace {

struct CurveOut {
  int32_t* idx;
  int64_t n;
  int width;
};

void curve_line(CurveOut& o, int x, int y, int dx, int dy, int len) {
  for (int i = 0; i < len; ++i) o.idx[o.n++] = (int32_t)((int64_t)(y + i * dy) * o.width + (x + i * dx));
}

void curve_block(CurveOut& o, int x, int y, int ax, int ay, int la, int bx, int by, int lb) {
  if (lb == 1) {
    curve_line(o, x, y, ax, ay, la);
    return;
  }
  if (la == 2) {
    curve_line(o, x, y, bx, by, lb);
    curve_line(o, x + ax + (lb - 1) * bx, y + ay + (lb - 1) * by, -bx, -by, lb);
    return;
  }
  if (la >= 2 * lb || lb == 2) {
    int a = la / 2;
    if (lb % 2 == 0 && a % 2 == 1) a = a - 1 >= 2 ? a - 1 : a + 1;
    curve_block(o, x, y, ax, ay, a, bx, by, lb);
    curve_block(o, x + a * ax, y + a * ay, ax, ay, la - a, bx, by, lb);
    return;
  }
  int b = lb / 2;
  if (b % 2 == 1) b = b + 1 <= lb - 1 ? b + 1 : b - 1;
  const int a = la / 2;
  curve_block(o, x, y, bx, by, b, ax, ay, a);
  curve_block(o, x + b * bx, y + b * by, ax, ay, la, bx, by, lb - b);
  curve_block(o, x + (la - 1) * ax + (b - 1) * bx, y + (la - 1) * ay + (b - 1) * by, -bx, -by, b, -ax, -ay,
              la - a);
}

}  // namespace

extern "C" avq_status avq_gilbert_order(int width, int height, int32_t* idx) {
  if (width < 1 || height < 1 || idx == nullptr || (int64_t)width * height > INT32_MAX)
    return AVQ_ERR_INVALID_ARG;
  CurveOut o{idx, 0, width};
  // start at (0, 0) and end at the next corner of the longer side when a path
  // along it exists (that side even, or both odd), else along the other side
  const bool along_x = width >= height ? (width % 2 == 0 || height % 2 == 1)
                                       : !(height % 2 == 0 || width % 2 == 1);
  if (along_x)
    curve_block(o, 0, 0, 1, 0, width, 0, 1, height);
  else
    curve_block(o, 0, 0, 0, 1, height, 1, 0, width);
  return o.n == (int64_t)width * height ? AVQ_OK : AVQ_ERR_INVALID_ARG;
}
