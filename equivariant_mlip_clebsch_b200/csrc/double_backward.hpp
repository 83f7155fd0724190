// double_backward.hpp -- the term structure of the double backward, on any
// forward/backward implementation (the library's kernels in capi.cpp; a host
// implementation in the tests).
//
// The convolution is linear in each of x, Y and W, so for cotangents
// (h_x, h_W, h_Y) of the backward's outputs
//   S = <g, fwd(h_x, Y, W) + fwd(x, Y, h_W) + fwd(x, h_Y, W)>,
// and the gradients of S are forwards and backwards with one argument
// replaced by its cotangent:
//   d g = fwd(h_x, Y, W) + fwd(x, Y, h_W) + fwd(x, h_Y, W)
//   d x = bwd_x(Y, h_W) + bwd_x(h_Y, W),   d W = bwd_W(h_x, Y) + bwd_W(x, h_Y),
//   d Y = bwd_Y(h_x, W) + bwd_Y(x, h_W).
// The first term of an output is written in place, later ones go through a
// scratch buffer and an add; an output no term reaches is zeroed.
#pragma once

#include <cstdint>

namespace cgtp {

struct DbwdDims {
  int64_t n_recv, n_send, E, D_in, D_e, D_out, U;
};

// Ops: forward(x, Y, W, out), backward(x, Y, W, gx, gW, gY) (null outputs not
// computed), add(dst, src, n) (dst += src), zero(dst, n); each returns 0 on
// success or an error code, which is returned as is.
template <class Ops>
int compose_double_backward(Ops& ops, const DbwdDims& d, const float* x, const float* Y, const float* W,
                            const float* h_x, const float* h_W, const float* h_Y, float* gg, float* gx,
                            float* gW, float* gY, float* tF, float* tX, float* tW, float* tY) {
  const float* tx[3] = {h_x, x, x};
  const float* ty[3] = {Y, Y, h_Y};
  const float* tw[3] = {W, h_W, W};
  const bool on[3] = {h_x != nullptr, h_W != nullptr, h_Y != nullptr};
  int st = 0;
  if (gg && d.n_recv > 0) {  // d S / d grad_out: the forwards
    bool written = false;
    for (int k = 0; k < 3; ++k) {
      if (!on[k]) continue;
      if ((st = ops.forward(tx[k], ty[k], tw[k], written ? tF : gg)) != 0) return st;
      if (written && (st = ops.add(gg, tF, d.n_recv * d.D_out)) != 0) return st;
      written = true;
    }
    if (!written && (st = ops.zero(gg, d.n_recv * d.D_out)) != 0) return st;
  }
  // d S / d (x, W, Y): term k gives the gradients of the two arguments it kept
  // (h_x: W and Y; h_W: x and Y; h_Y: x and W)
  bool wx = false, ww = false, wy = false;
  for (int k = 0; k < 3; ++k) {
    if (!on[k]) continue;
    float* ox = (k != 0 && gx) ? (wx ? tX : gx) : nullptr;
    float* ow = (k != 1 && gW) ? (ww ? tW : gW) : nullptr;
    float* oy = (k != 2 && gY) ? (wy ? tY : gY) : nullptr;
    if (!ox && !ow && !oy) continue;
    if ((st = ops.backward(tx[k], ty[k], tw[k], ox, ow, oy)) != 0) return st;
    if (ox == tX && (st = ops.add(gx, tX, d.n_send * d.D_in)) != 0) return st;
    if (ow == tW && (st = ops.add(gW, tW, d.E * d.U)) != 0) return st;
    if (oy == tY && (st = ops.add(gY, tY, d.E * d.D_e)) != 0) return st;
    wx = wx || ox;
    ww = ww || ow;
    wy = wy || oy;
  }
  if (gx && !wx && d.n_send > 0 && (st = ops.zero(gx, d.n_send * d.D_in)) != 0) return st;
  if (gW && !ww && d.E > 0 && (st = ops.zero(gW, d.E * d.U)) != 0) return st;
  if (gY && !wy && d.E > 0 && (st = ops.zero(gY, d.E * d.D_e)) != 0) return st;
  return 0;
}

}  // namespace cgtp
