// codegen_bwd.cpp -- the backward CGTP convolution kernel, generated per plan.
//
// Given g = dL/dout (LunaTP, arXiv 2610.18393, Table 11 lists the backward
// outputs x-bar, y-bar, w-bar), per edge e = (i <- j) and path p, channel u:
//   t[m3]  = sum_m1 Chat[m3][m1] x[j][u][m1]            (as in the forward)
//   dW[e][k0+u]      = sum_m3 g[i][u][m3] t[m3]
//   h[m3]  = W[e][k0+u] g[i][u][m3]
//   msg[e][u][m1]   += sum_m3 Chat[m3][m1] h[m3]        (summed over the paths of the irrep)
//   dY[e][l2^2+m2]  += sum_{u,m1,m3} C[m1][m2][m3] x[j][u][m1] h[m3]
// and dx[j] = sum over the edges leaving j of msg[e] (a second, sender-major
// pass over the transpose edge list, in kernels.cu).
//
// Execution: grid (n_recv, S), receiver-major like the forward.  The
// receiver's g row (its slice) is staged in shared memory once; W, x and Y of
// the edges stream through the same bulk-copy ring as the forward.  A warp
// role owns R channels per lane of one hidden irrep, ALL paths of that irrep
// (so msg is complete in registers) and the edges b of each chunk with
// b % nph == ph.  dW and msg are written straight to global memory; the dY
// partial of each role is reduced across the warp by shuffles and across the
// roles of the CTA in a fixed order through shared memory, so the result is
// bitwise reproducible.  With S > 1 slices the per-slice dY parts go to the
// workspace and are summed by a small kernel.
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <numeric>
#include <sstream>

#include "codegen_common.hpp"

namespace cgtp {

namespace {

int path_nnz(const Plan& P, int pi) {
  const Path& p = P.paths[pi];
  const int n = (2 * p.l1 + 1) * (2 * p.l2 + 1) * (2 * p.l3 + 1);
  int c = 0;
  for (int t = 0; t < n; ++t) c += P.coeff[p.c_off + t] != 0.0;
  return c;
}

std::string flt(double v) {
  char b[48];
  std::snprintf(b, sizeof b, "%.9ef", (double)(float)v);
  return b;
}

}  // namespace

static std::string gen_bwd_source(const Plan& P, const std::vector<SliceLayout>& SL,
                                  const std::string& kname, int& smem_bytes) {
  const FwdConfig& F = P.bcfg;
  const int S = F.S, NW = F.nw, B = F.B;
  int GS = 0;
  for (const auto& sl : SL) GS = std::max(GS, sl.gs);
  auto r128 = [](int v) { return (v + 127) & ~127; };
  const int extra = r128(GS * 4) + r128(NW * B * (int)P.D_e * 4);
  int off_g = 0;
  std::ostringstream o;
  o << kPrelude;
  o << gen_layout(P, F, SL, extra, off_g, smem_bytes);
  o << "#define OFF_G " << off_g << "\n#define OFF_DY " << off_g + r128(GS * 4) << "\n";
  o << gen_slice_helpers(P, F, SL);
  o << gen_producer(P, F);

  // g staging per slice (by the consumer threads)
  o << "__device__ __forceinline__ void stage_g(int s, const float* __restrict__ grow, float* sg, int tid) {\n"
       "  switch (s) {\n";
  for (int s = 0; s < S; ++s) {
    o << "  case " << s << ":\n";
    std::vector<std::array<int, 3>> cp;
    for (int pi : SL[s].paths) {
      const Path& p = P.paths[pi];
      const int src = p.o_off, dst = SL[s].g_st.at(pi), n = p.mul * (2 * p.l3 + 1);
      if (!cp.empty() && cp.back()[0] + cp.back()[2] == src && cp.back()[1] + cp.back()[2] == dst)
        cp.back()[2] += n;
      else
        cp.push_back({src, dst, n});
    }
    for (auto& c : cp)
      o << "    for (int t = tid; t < " << c[2] << "; t += NW * 32) sg[" << c[1] << " + t] = grow[" << c[0]
        << " + t];\n";
    o << "    break;\n";
  }
  o << "  }\n}\n";
  // per-slot phase tables and the fixed-order dY reduction over the roles
  o << "__device__ const int kPh[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? P.bwd_roles[F.slice_roles[s][w]].ph : -1) << ",";
  o << "};\n__device__ const int kNph[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? P.bwd_roles[F.slice_roles[s][w]].nph : 1) << ",";
  o << "};\n";
  o << "__device__ __forceinline__ void dy_reduce(const float* __restrict__ sdyall, float* __restrict__ dys,\n"
       "    int slice, int eb, int nb) {\n"
       "  for (int t = threadIdx.x; t < nb * DE; t += NW * 32) {\n"
       "    const int b = t / DE, k = t - b * DE;\n"
       "    float v = 0.f;\n"
       "    for (int w = 0; w < NW; ++w) {\n"
       "      const int ph = kPh[slice * NW + w];\n"
       "      if (ph >= 0 && b % kNph[slice * NW + w] == ph) v += sdyall[(w * NB + b) * DE + k];\n"
       "    }\n"
       "    dys[(size_t)(eb + b) * DE + k] = v;\n"
       "  }\n"
       "}\n";

  // one consumer function per (irrep, R); channel block and phase at run time
  std::vector<int> shape_of(P.bwd_roles.size(), -1), shape_rep;
  std::vector<int> slice_of(P.bwd_roles.size(), -1);
  for (int s = 0; s < S; ++s)
    for (int v : F.slice_roles[s]) slice_of[v] = s;
  for (size_t ri = 0; ri < P.bwd_roles.size(); ++ri) {
    const BwdRole& r = P.bwd_roles[ri];
    for (size_t k = 0; k < shape_rep.size(); ++k) {
      const BwdRole& q = P.bwd_roles[shape_rep[k]];
      if (q.irrep == r.irrep && q.R == r.R && slice_of[shape_rep[k]] == slice_of[ri]) {
        shape_of[ri] = (int)k;
        break;
      }
    }
    if (shape_of[ri] < 0) {
      shape_of[ri] = (int)shape_rep.size();
      shape_rep.push_back((int)ri);
    }
  }
  const std::string loop_head =
      "  const int lane = threadIdx.x & 31;\n"
      "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
      "  const int nchunk = (e1 - e0 + NB - 1) / NB;\n"
      "  float* sdyall = reinterpret_cast<float*>(smem + OFF_DY);\n"
      "  bool dead = false;\n"
      "  for (int c = 0; c < nchunk; ++c) {\n"
      "    const int s = c % NSTAGE;\n"
      "    if (!dead && !mbar_wait(full0 + 8 * s, (c / NSTAGE) & 1)) { dead = true; if (lane == 0) atomicOr(err, 10); }\n"
      "    const int eb = e0 + c * NB;\n"
      "    const int nb = min(NB, e1 - eb);\n"
      "    unsigned char* st = smem + OFF_STAGE + s * STAGE_BYTES;\n"
      "    const float* sY = reinterpret_cast<const float*>(st + W_BYTES + X_BYTES);\n"
      "    float* ch = reinterpret_cast<float*>(smem + OFF_CH) + (c & 1) * NB * CHS;\n"
      "    if (!dead) chat_build(sent, nent, term, sY, ch, chs, nb, threadIdx.x);\n"
      "    consumer_bar(NW * 32);\n";
  const std::string loop_tail =
      "    consumer_bar(NW * 32);\n"
      "    if (!dead && dys) dy_reduce(sdyall, dys, slice, eb, nb);\n"
      "    __syncwarp();\n"
      "    if (lane == 0) mbar_arrive(empty0 + 8 * s);\n"
      "  }\n";
  const std::string params =
      "(const int* __restrict__ col, const float* __restrict__ x, const float* __restrict__ W,\n"
      "    float* __restrict__ dW, float* __restrict__ msg, float* __restrict__ dys,\n"
      "    const int4* __restrict__ sent, int nent, const int2* __restrict__ term, int* __restrict__ err,\n"
      "    unsigned char* smem, const float* __restrict__ sg, int slice, int e0, int e1, int u0, int ph,\n"
      "    int nph, int chs)";
  for (size_t k = 0; k < shape_rep.size(); ++k) {
    const BwdRole& r = P.bwd_roles[shape_rep[k]];
    const SliceLayout& sl = SL[slice_of[shape_rep[k]]];
    const Irrep& h = P.in[r.irrep];
    const int N1 = 2 * h.l + 1, R = r.R, MUL = h.mul;
    const int xoff = F.x_smem ? sl.x_st.at(r.irrep) : P.x_off[r.irrep];
    std::vector<int> ps;
    for (size_t q = 0; q < P.paths.size(); ++q)
      if (P.paths[q].irrep == r.irrep) ps.push_back((int)q);
    o << "// shape " << k << ": irrep " << r.irrep << " (" << h.mul << "x" << h.l << "), R=" << R << ", "
      << ps.size() << " paths\n";
    o << "__device__ __noinline__ void bcons_" << k << params << " {\n" << loop_head;
    o << "    bool ok[" << R << "];\n"
      << "#pragma unroll\n    for (int r = 0; r < " << R << "; ++r) ok[r] = u0 + r * 32 + lane < " << MUL << ";\n"
      << "    if (!dead) {\n"
      << "      for (int b = ph; b < nb; b += nph) {\n"
      << "        const int e = eb + b;\n";
    if (F.w_smem)
      o << "        const float* wr = reinterpret_cast<const float*>(st) + b * NU;\n";
    else
      o << "        const float* wr = W + (size_t)e * NU;\n";
    if (F.x_smem)
      o << "        const float* xr = reinterpret_cast<const float*>(st + W_BYTES) + b * XS + " << xoff << ";\n";
    else
      o << "        const float* xr = x + (size_t)col[e] * DIN + " << xoff << ";\n";
    o << "        const float* chb = ch + b * chs;\n"
      << "        float* dWrow = dW ? dW + (size_t)e * NU : nullptr;\n"
      << "        float* sdy = dys ? sdyall + ((threadIdx.x >> 5) * NB + b) * DE : nullptr;\n"
      << "        float xv[" << R << "][" << N1 << "], mx[" << R << "][" << N1 << "];\n"
      << "#pragma unroll\n        for (int r = 0; r < " << R << "; ++r) {\n"
      << "          const int u = u0 + r * 32 + lane;\n"
      << "#pragma unroll\n          for (int m1 = 0; m1 < " << N1
      << "; ++m1) { mx[r][m1] = 0.f; xv[r][m1] = ok[r] ? LDX(xr + u * " << N1 << " + m1) : 0.f; }\n"
      << "        }\n";
    std::vector<char> l2seen(P.L + 1, 0);
    size_t q = 0;
    while (q < ps.size()) {
      const int l2 = P.paths[ps[q]].l2;
      const int N2 = 2 * l2 + 1;
      l2seen[l2] = 1;
      o << "        {\n          float z[" << N2 << "];\n#pragma unroll\n          for (int t = 0; t < " << N2
        << "; ++t) z[t] = 0.f;\n";
      for (; q < ps.size() && P.paths[ps[q]].l2 == l2; ++q) {
        const int pi = ps[q];
        const Path& p = P.paths[pi];
        const int N3 = 2 * p.l3 + 1, n2 = 2 * p.l2 + 1;
        o << "          {\n            float w[" << R << "], gv[" << R << "][" << N3 << "], hh[" << R << "][" << N3
          << "], dw[" << R << "];\n"
          << "#pragma unroll\n            for (int r = 0; r < " << R << "; ++r) {\n"
          << "              const int u = u0 + r * 32 + lane;\n"
          << "              w[r] = ok[r] ? LDW(wr + " << p.k0 << " + u) : 0.f;\n"
          << "#pragma unroll\n              for (int m3 = 0; m3 < " << N3 << "; ++m3) gv[r][m3] = ok[r] ? sg["
          << sl.g_st.at(pi) << " + u * " << N3 << " + m3] : 0.f;\n            }\n"
          << "            bpath<" << N1 << "," << N3 << "," << R << ">(chb + " << sl.ch_off.at(pi)
          << ", xv, w, gv, hh, mx, dw);\n"
          << "            if (dWrow) {\n#pragma unroll\n              for (int r = 0; r < " << R
          << "; ++r) if (ok[r]) dWrow[" << p.k0 << " + u0 + r * 32 + lane] = dw[r];\n            }\n"
          << "            if (sdy) {\n#pragma unroll\n              for (int r = 0; r < " << R << "; ++r) {\n";
        const double* C = P.coeff.data() + p.c_off;
        for (int m1 = 0; m1 < N1; ++m1)
          for (int m3 = 0; m3 < N3; ++m3) {
            std::vector<std::pair<int, double>> t;
            for (int m2 = 0; m2 < n2; ++m2) {
              const double c = C[((size_t)m1 * n2 + m2) * N3 + m3];
              if (c != 0.0) t.push_back({m2, c});
            }
            if (t.empty()) continue;
            o << "                { const float pr = xv[r][" << m1 << "] * hh[r][" << m3 << "];";
            for (auto& tc : t)
              o << " z[" << tc.first << "] = fmaf(" << flt(tc.second) << ", pr, z[" << tc.first << "]);";
            o << " }\n";
          }
        o << "              }\n            }\n          }\n";
      }
      o << "          if (sdy) {\n#pragma unroll\n            for (int t = 0; t < " << N2
        << "; ++t) { const float v = warp_sum(z[t]); if (lane == 0) sdy[" << l2 * l2 << " + t] = v; }\n"
        << "          }\n        }\n";
    }
    for (int l2 = 0; l2 <= P.L; ++l2)
      if (!l2seen[l2])
        o << "        if (sdy && lane == 0) {\n#pragma unroll\n          for (int t = 0; t < " << 2 * l2 + 1
          << "; ++t) sdy[" << l2 * l2 << " + t] = 0.f;\n        }\n";
    o << "        if (msg) {\n#pragma unroll\n          for (int r = 0; r < " << R
      << "; ++r) if (ok[r]) {\n            const int u = u0 + r * 32 + lane;\n"
      << "#pragma unroll\n            for (int m1 = 0; m1 < " << N1 << "; ++m1) msg[(size_t)e * DIN + "
      << P.x_off[r.irrep] << " + u * " << N1 << " + m1] = mx[r][m1];\n          }\n        }\n";
    o << "      }\n    }\n" << loop_tail << "}\n";
  }
  o << "__device__ __noinline__ void bcons_idle" << params << " {\n" << loop_head << loop_tail << "}\n";

  o << "__device__ const int kShape[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? shape_of[F.slice_roles[s][w]] : -1) << ",";
  o << "};\n__device__ const int kU0[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? P.bwd_roles[F.slice_roles[s][w]].u0 : 0) << ",";
  o << "};\n__device__ const int kEntBegin[" << S + 1 << "] = {";
  for (int v : P.bwd_ent_begin) o << v << ",";
  o << "};\n";
  o << "extern \"C\" __global__ void __launch_bounds__((NW + 1) * 32) " << kname
    << "(const int* __restrict__ rowptr, const int* __restrict__ col, const float* __restrict__ x,\n"
       "    const float* __restrict__ Y, const float* __restrict__ W, const float* __restrict__ g,\n"
       "    float* __restrict__ dW, float* __restrict__ dyp, float* __restrict__ msg,\n"
       "    const int4* __restrict__ ent, const int2* __restrict__ term, int* __restrict__ err) {\n"
       "  extern __shared__ __align__(128) unsigned char smem[];\n"
       "  const int i = blockIdx.x, slice = blockIdx.y;\n"
       "  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;\n"
       "  const int e0 = rowptr[i], e1 = rowptr[i + 1];\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  if (threadIdx.x == 0) {\n"
       "    for (int s = 0; s < NSTAGE; ++s) { mbar_init(full0 + 8 * s, 32); mbar_init(empty0 + 8 * s, NW); }\n"
       "    fence_mbar_init();\n"
       "  }\n"
       "  __syncthreads();\n"
       "  if (e1 == e0) return;\n"
       "  if (warp == NW) { producer(col, x, Y, W, err, smem, slice, e0, e1, lane); return; }\n"
       "  float* sg = reinterpret_cast<float*>(smem + OFF_G);\n"
       "  stage_g(slice, g + (size_t)i * DOUT, sg, threadIdx.x);\n"
       "  const int E = rowptr[gridDim.x];\n"
       "  float* dys = dyp ? dyp + (size_t)slice * E * DE : nullptr;\n"
       "  const int4* sent = ent + kEntBegin[slice];\n"
       "  const int nent = kEntBegin[slice + 1] - kEntBegin[slice];\n"
       "  const int chs = slice_chs(slice);\n"
       "  const int slot = slice * NW + warp;\n"
       "  const int u0 = kU0[slot], ph = kPh[slot], nph = kNph[slot];\n"
       "  switch (kShape[slot]) {\n";
  for (size_t k = 0; k < shape_rep.size(); ++k)
    o << "  case " << k << ": bcons_" << k
      << "(col, x, W, dW, msg, dys, sent, nent, term, err, smem, sg, slice, e0, e1, u0, ph, nph, chs); break;\n";
  o << "  default: bcons_idle(col, x, W, dW, msg, dys, sent, nent, term, err, smem, sg, slice, e0, e1, u0, ph, nph, chs); break;\n"
       "  }\n}\n";
  return o.str();
}

cgtp_status build_backward(Plan& P) {
  P.bwd_roles.clear();
  FwdConfig& F = P.bcfg;
  F = FwdConfig();
  if (P.paths.empty()) return CGTP_OK;
  // cost of one channel block of each irrep per edge
  struct IrrepWork {
    int a, R, nblk;
    double cost;
  };
  std::vector<IrrepWork> iw;
  double total = 0.0;
  for (size_t a = 0; a < P.in.size(); ++a) {
    const Irrep& h = P.in[a];
    const int n1 = 2 * h.l + 1;
    double c = 0.0;
    bool any = false;
    for (size_t k = 0; k < P.paths.size(); ++k)
      if (P.paths[k].irrep == (int)a) {
        const int n3 = 2 * P.paths[k].l3 + 1;
        c += 2.0 * n1 * n3 + 3.0 * n3 + 2.0 * path_nnz(P, (int)k);
        any = true;
      }
    if (!any) {
      P.bwd_irrep_gap = true;
      continue;
    }
    const int R = (h.mul >= 64 && h.l <= 3) ? 2 : 1;
    const int nblk = (h.mul + 32 * R - 1) / (32 * R);
    iw.push_back({(int)a, R, nblk, c * R});
    total += nblk * c * R;
  }
  const int kMaxWarps = 16;
  int maxnph = 4;
  std::vector<SliceLayout> SL;
  for (int attempt = 0; attempt < 3; ++attempt) {
    P.bwd_roles.clear();
    const double tau = total / kMaxWarps;
    const bool fits_one = (long)P.D_out * 4 <= 64 * 1024;
    for (auto& w : iw) {
      int nph = fits_one ? (int)std::lround(w.cost / std::max(tau, 1e-9))
                         : std::max(1, 8 / w.nblk);
      nph = std::max(1, std::min(maxnph, nph));
      while (nph & (nph - 1)) --nph;  // 1, 2 or 4
      for (int blk = 0; blk < w.nblk; ++blk)
        for (int ph = 0; ph < nph; ++ph) {
          BwdRole r;
          r.irrep = w.a;
          r.u0 = blk * 32 * w.R;
          r.R = w.R;
          r.ph = ph;
          r.nph = nph;
          r.cost = w.cost / nph;
          P.bwd_roles.push_back(r);
        }
    }
    const int NR = (int)P.bwd_roles.size();
    // one slice holding every role when it fits in a CTA (the receiver's
    // whole g row staged once), otherwise one slice per hidden irrep
    const bool one = NR <= kMaxWarps && (long)P.D_out * 4 <= 64 * 1024;
    F.slice_roles.clear();
    if (one) {
      F.slice_roles.assign(1, {});
      for (int ri = 0; ri < NR; ++ri) F.slice_roles[0].push_back(ri);
    } else {
      for (auto& w : iw) {
        F.slice_roles.push_back({});
        for (int ri = 0; ri < NR; ++ri)
          if (P.bwd_roles[ri].irrep == w.a) F.slice_roles.back().push_back(ri);
      }
    }
    F.S = (int)F.slice_roles.size();
    for (auto& v : F.slice_roles) std::sort(v.begin(), v.end());
    F.nw = 0;
    for (auto& v : F.slice_roles) F.nw = std::max<int>(F.nw, (int)v.size());
    // layouts
    SL.assign(F.S, SliceLayout());
    for (int s = 0; s < F.S; ++s) {
      SliceLayout& sl = SL[s];
      std::vector<char> iseen(P.in.size(), 0);
      for (int ri : F.slice_roles[s]) iseen[P.bwd_roles[ri].irrep] = 1;
      for (size_t k = 0; k < P.paths.size(); ++k)
        if (iseen[P.paths[k].irrep]) {
          sl.paths.push_back((int)k);
          sl.ch_off[(int)k] = sl.chs;
          sl.chs += chat_size(P.paths[k].l1, P.paths[k].l3);
        }
      for (size_t a = 0; a < P.in.size(); ++a)
        if (iseen[a]) {
          sl.irreps.push_back((int)a);
          sl.x_st[(int)a] = sl.xs;
          sl.xs += pad4(P.in[a].mul * (2 * P.in[a].l + 1));
        }
      // g blocks: with every path of the plan in the slice, the row is copied
      // as is; otherwise the slice's path blocks are packed
      if (sl.paths.size() == P.paths.size()) {
        for (int pi : sl.paths) sl.g_st[pi] = P.paths[pi].o_off;
        sl.gs = (int)P.D_out;
      } else {
        for (int pi : sl.paths) {
          sl.g_st[pi] = sl.gs;
          sl.gs += P.paths[pi].mul * (2 * P.paths[pi].l3 + 1);
        }
      }
    }
    F.w_smem = (F.S == 1) && (P.U % 4 == 0);
    F.x_smem = (P.D_in % 4 == 0);
    for (int s = 0; s < F.S && F.x_smem; ++s)
      for (int a : SL[s].irreps)
        if (P.x_off[a] % 4 != 0 || (P.in[a].mul * (2 * P.in[a].l + 1)) % 4 != 0) F.x_smem = false;
    if (!F.x_smem)
      for (auto& sl : SL) {
        sl.xs = 0;
        for (int a : sl.irreps) sl.x_st[a] = P.x_off[a];
      }
    int CHS = 0, XS = 0, GS = 0;
    for (auto& sl : SL) {
      CHS = std::max(CHS, sl.chs);
      XS = std::max(XS, sl.xs);
      GS = std::max(GS, sl.gs);
    }
    const long pe = (F.w_smem ? P.U * 4 : 0) + (F.x_smem ? XS * 4 : 0) + P.D_e * 4 + 64;
    const long fixed = (long)GS * 4 + 1024;
    const long budget = std::max<long>(100 * 1024, fixed + 40 * 1024);
    F.B = 4;
    auto per_b = [&](int b) { return 2L * b * CHS * 4 + (long)F.nw * b * P.D_e * 4 + 2L * b * pe; };
    while (F.B > 1 && fixed + per_b(F.B) > budget) F.B /= 2;
    F.stages = (int)std::min<long>(
        8, std::max<long>(2, (budget - fixed - 2L * F.B * CHS * 4 - (long)F.nw * F.B * P.D_e * 4) /
                                 (F.B * pe)));
    if (F.B >= maxnph) break;
    maxnph = F.B;
  }

  cgtp_status st = upload_chat_tables(P, SL, &P.d_bwd_ent, &P.d_bwd_term, P.bwd_ent_begin);
  if (st != CGTP_OK) return st;
  int smem = 0;
  const std::string name = "cgtp_bwd";
  std::string src = gen_bwd_source(P, SL, name, smem);
  if (smem > 227 * 1024) return fail(CGTP_ERR_SIZE, "backward kernel needs too much shared memory");
  P.bwd.threads = (F.nw + 1) * 32;
  P.bwd.smem = smem;
  if (const char* d = std::getenv("CGTP_DUMP_SOURCE")) {
    FILE* f = std::fopen((std::string(d) + "/bwd.cu").c_str(), "w");
    if (f) {
      std::fputs(src.c_str(), f);
      std::fclose(f);
    }
  }
  return jit_compile(src, name, P.bwd);
}

}  // namespace cgtp
