// codegen_bwd.cpp -- the backward CGTP convolution kernel, generated per plan.
//
// Given g = dL/dout (LunaTP, arXiv 2610.18393, Table 11 lists the backward
// outputs x-bar, y-bar, w-bar), per edge e = (i <- j), path p, channel u,
// with Chat[m3][m1] = sum_m2 C[m1][m2][m3] Y[e][l2^2+m2]:
//   s[m1]  = sum_m3 Chat[m3][m1] g[i][u][m3]
//   dW[e][k0+u]      = sum_m1 x[j][u][m1] s[m1]   (= sum_m3 g (Chat x)[m3])
//   msg[e][u][m1]   += W[e][k0+u] s[m1]           (over the paths of the irrep)
//   dY[e][l2^2+m2]  += sum_{u,m1,m3} C[m1][m2][m3] W[e][k0+u] x[j][u][m1] g[i][u][m3]
// and dx[j] = sum over the edges leaving j of msg[e] (a second, sender-major
// pass over the transpose edge list, kernels.cu).  The default roles form
// these "CG first" (gen_bwd_role_cg_first: t = C g per channel, then s and
// the dY partial from t and Y, no Chat); the staged-Chat roles (the helper
// builds Chat per edge in shared memory) remain behind CGTP_BWD_TFORM=0.
//
// Execution: persistent CTAs (resident CTAs per SM x SMs) walk the slices
// in turn; a slice is a group of hidden irreps, chosen with the chunk size and
// warp count by the planner (build_backward).  Within a slice the TMA warp
// stages each receiver's grad_out pieces once and, per chunk, the W and x
// pieces of the slice; the helper warp stages Y (and builds Chat for the
// staged-Chat roles) and sums the dY partials of released stages.  A
// consumer owns R blocks of 32 channels of one
// irrep (run one after another), ALL its paths (so msg is complete in
// registers) and the edges b of each chunk with b % nph == ph.  Two variants
// are compiled: CTAs over receivers blockIdx.x, + gridDim.x, ..., and CTAs
// over equal edge ranges (for graphs with few receivers per CTA).  dW and msg
// go straight to global memory; dY partials are reduced over lanes by
// shuffles, over the CTA's warps by the helper in a fixed order, and over
// slices by the closing reduction kernel: bitwise reproducible.
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <functional>
#include <numeric>
#include <sstream>
#include <thread>

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

// Channel blocks of a backward role unrolled together.  One: measured on
// B200, unrolling two or four blocks (for l <= 1 inputs) was slower overall
// than running every block in the loop, whose code is the smallest.
int bwd_unroll(int n1, int R) {
  (void)n1;
  (void)R;
  return 1;
}

std::string flt(double v) {
  char b[48];
  std::snprintf(b, sizeof b, "%.9ef", (double)(float)v);
  return b;
}

// One consumer role of the CG-first backward (no staged Chat).  Per path and
// channel, with g = grad_out of the receiver:
//   t[m1][m2] = sum_m3 C[m1][m2][m3] g[m3]      (CG coefficients as immediates)
//   s[m1]     = sum_m2 Y[m2] t[m1][m2]           (= sum_m3 Chat[m3][m1] g[m3])
//   dW += x[m1] s[m1],  msg[m1] += w s[m1],  dY[m2] += w x[m1] t[m1][m2].
// The tangent form (double backward) adds the directional derivatives along
// (xt, Yt, wt): st = sum_m2 Yt t, dW += xt s + x st, msg += wt s + w st and
// dY += (w xt + wt x) t.
void gen_bwd_role_cg_first(std::ostream& o, const Plan& P, const KernelShape& K, const BwdRole& r,
                           const SliceLayout& sl, size_t k, const std::string& params) {
  const Irrep& h = P.in[r.irrep];
  const int N1 = 2 * h.l + 1, R = r.R, MUL = h.mul;
  const bool tan = K.tangent;
  auto pow2 = [](int n) { int v = 1; while (v < n) v <<= 1; return v; };
  const bool combined = P.D_e <= 32;
  if (!combined && R != 1) {
    std::fprintf(stderr, "cgtp: backward role with R > 1 needs D_e <= 32\n");
    std::abort();
  }
  const int VZ = (int)P.D_e;
  std::vector<int> ps;
  for (size_t q = 0; q < P.paths.size(); ++q)
    if (P.paths[q].irrep == r.irrep) ps.push_back((int)q);
  const std::string sN1 = std::to_string(N1);
  o << "// shape " << k << ": irrep " << r.irrep << " (" << h.mul << "x" << h.l << "), R=" << R << ", " << ps.size()
    << " paths, CG first\n"
    << "__device__ __noinline__ void bcons_" << k << params << " {\n"
    << "  const int lane = threadIdx.x & 31;\n"
    << "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
    << "  const u32 gfull0 = full0 + OFF_GFULL, gempty0 = full0 + OFF_GEMPTY;\n"
    << "  (void)chs;\n"
    << "  int q = *qp, kr = *kp;\n"
    << "#pragma unroll 1\n  for (int i = RECV_FIRST; i < RECV_END; i += RECV_STEP) {\n"
    << "  const int e0 = EDGE_LO(i), e1 = EDGE_HI(i);\n"
    << "  if (e1 <= e0) continue;\n"
    << "  const int gb = kr % GBUF;\n"
    << "  if (!mbar_wait(gfull0 + 8 * gb, (kr / GBUF) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
    << "  const float* sg = reinterpret_cast<const float*>(smem + OFF_G) + gb * GS;\n"
    << "#pragma unroll 1\n  for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
    << "    const int s = q % NSTAGE;\n"
    << "    if (!stage_ready(full0, s, (q / NSTAGE) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
    << "    const int nb = min(NB, e1 - eb);\n"
    << "    unsigned char* st = stage_ptr(smem, s);\n"
    << "    float* sdyw = reinterpret_cast<float*>(st + OFF_DY) + (threadIdx.x >> 5) * NB * DE;\n"
    << "#pragma unroll 1\n    for (int b = ph; b < nb; b += nph) {\n"
    << "      const int e = eb + b;\n"
    << "      const float* wr = reinterpret_cast<const float*>(st + OFF_W) + b * WS;\n"
    << "      const float* xr = reinterpret_cast<const float*>(st + OFF_X) + " << sl.x_st.at(r.irrep) << " + b * XS;\n"
    << "      const float* yr = reinterpret_cast<const float*>(st + OFF_Y) + b * DE;\n"
    << (tan ? "      const float* wtr = reinterpret_cast<const float*>(st + OFF_WT) + b * WS;\n"
              "      const float* xtr = reinterpret_cast<const float*>(st + OFF_XT) + " +
                  std::to_string(sl.x_st.at(r.irrep)) +
                  " + b * XS;\n"
                  "      const float* ytr = reinterpret_cast<const float*>(st + OFF_YT) + b * DE;\n"
            : "")
    << "      float* dWrow = dW ? dW + (size_t)(eid ? __ldg(eid + e) : e) * NU : nullptr;\n"
    << "      float* sdy = want_dy ? sdyw + b * DE : nullptr;\n";
  if (combined)
    o << "      float z[" << VZ << "];\n#pragma unroll\n      for (int t = 0; t < " << VZ << "; ++t) z[t] = 0.f;\n";
  o << "#pragma unroll 1\n      for (int r = 0; r < " << R << "; ++r) {\n"
    << "      const int u = u0 + r * 32 + lane;\n"
    << "      const bool ok = " << (MUL % (32 * R) == 0 ? std::string("true") : "u < " + std::to_string(MUL))
    << ";  // every lane holds a channel when the blocks are full\n"
    << "      float xv[" << N1 << "], mx[" << N1 << "];\n"
    << (tan ? "      float xtv[" + sN1 + "];\n" : "")
    << "#pragma unroll\n      for (int m1 = 0; m1 < " << N1 << "; ++m1) {\n"
    << "        mx[m1] = 0.f;\n"
    << "        xv[m1] = ok ? xr[u * " << N1 << " + m1] : 0.f;\n"
    << (tan ? "        xtv[m1] = ok ? xtr[u * " + sN1 + " + m1] : 0.f;\n" : "")
    << "      }\n";
  std::vector<char> l2seen(P.L + 1, 0);
  size_t q = 0;
  while (q < ps.size()) {
    const int l2 = P.paths[ps[q]].l2;
    const int N2 = 2 * l2 + 1;
    const int zo = combined ? l2 * l2 : 0;  // offset of degree l2 inside z
    l2seen[l2] = 1;
    o << "      {\n";
    if (!combined)
      o << "        float z[" << pow2(N2) << "];\n#pragma unroll\n        for (int t = 0; t < " << pow2(N2)
        << "; ++t) z[t] = 0.f;\n";
    // this degree's harmonics of the edge (the same for every lane)
    o << "        float yl[" << N2 << "];\n#pragma unroll\n        for (int m2 = 0; m2 < " << N2
      << "; ++m2) yl[m2] = yr[" << l2 * l2 << " + m2];\n";
    if (tan)
      o << "        float ytl[" << N2 << "];\n#pragma unroll\n        for (int m2 = 0; m2 < " << N2
        << "; ++m2) ytl[m2] = ytr[" << l2 * l2 << " + m2];\n";
    for (; q < ps.size() && P.paths[ps[q]].l2 == l2; ++q) {
      const int pi = ps[q];
      const Path& p = P.paths[pi];
      const int N3 = 2 * p.l3 + 1, n2 = 2 * p.l2 + 1;
      o << "        {\n          float gv[" << N3 << "];\n"
        << "#pragma unroll\n          for (int m3 = 0; m3 < " << N3 << "; ++m3) gv[m3] = ok ? sg[" << sl.g_st.at(pi)
        << " + u * " << N3 << " + m3] : 0.f;\n"
        << "          const float w = ok ? wr[" << sl.w_st.at(pi) << " + u] : 0.f;\n"
        << (tan ? "          const float wt = ok ? wtr[" + std::to_string(sl.w_st.at(pi)) + " + u] : 0.f;\n" : "")
        << "          float d = 0.f;\n";
      const double* C = P.coeff.data() + p.c_off;
      for (int m1 = 0; m1 < N1; ++m1) {
        std::vector<int> m2s;
        std::ostringstream tdef;
        for (int m2 = 0; m2 < n2; ++m2) {
          std::vector<std::pair<int, double>> t;
          for (int m3 = 0; m3 < N3; ++m3) {
            const double c = C[((size_t)m1 * n2 + m2) * N3 + m3];
            if (c != 0.0) t.push_back({m3, c});
          }
          if (t.empty()) continue;
          m2s.push_back(m2);
          std::string e = flt(t[0].second) + " * gv[" + std::to_string(t[0].first) + "]";
          for (size_t c = 1; c < t.size(); ++c)
            e = "fmaf(" + flt(t[c].second) + ", gv[" + std::to_string(t[c].first) + "], " + e + ")";
          tdef << "            const float t" << m2 << " = " << e << ";\n";
        }
        if (m2s.empty()) continue;
        auto dot = [&](const std::string& y) {
          std::string e = y + "[" + std::to_string(m2s[0]) + "] * t" + std::to_string(m2s[0]);
          for (size_t c = 1; c < m2s.size(); ++c)
            e = "fmaf(" + y + "[" + std::to_string(m2s[c]) + "], t" + std::to_string(m2s[c]) + ", " + e + ")";
          return e;
        };
        const std::string xm = "xv[" + std::to_string(m1) + "]", mm = "mx[" + std::to_string(m1) + "]";
        o << "          {\n" << tdef.str() << "            const float s = " << dot("yl") << ";\n";
        if (tan) {
          const std::string xt = "xtv[" + std::to_string(m1) + "]";
          o << "            const float st = " << dot("ytl") << ";\n"
            << "            d = fmaf(" << xt << ", s, fmaf(" << xm << ", st, d));\n"
            << "            " << mm << " = fmaf(wt, s, fmaf(w, st, " << mm << "));\n"
            << "            const float wx = fmaf(w, " << xt << ", wt * " << xm << ");\n";
        } else {
          o << "            d = fmaf(" << xm << ", s, d);\n"
            << "            " << mm << " = fmaf(w, s, " << mm << ");\n"
            << "            const float wx = w * " << xm << ";\n";
        }
        for (int m2 : m2s)
          o << "            z[" << zo + m2 << "] = fmaf(wx, t" << m2 << ", z[" << zo + m2 << "]);\n";
        o << "          }\n";
      }
      o << "          if (dWrow && ok) dWrow[" << p.k0 << " + u] = d;\n        }\n";
    }
    if (!combined) {
      const int V = pow2(N2), LV = __builtin_ctz(V), sh = 5 - LV;
      o << "        if (sdy) {\n          const float v = warp_sum_many<" << V << ">(z, lane);\n"
        << "          const int c = lane >> " << sh << ";\n"
        << "          if ((lane & " << ((1 << sh) - 1) << ") == 0 && c < " << N2 << ") sdy[" << l2 * l2
        << " + c] = v;\n        }\n";
    }
    o << "      }\n";
  }
  // the message row segment of this channel block, through the warp's buffer
  o << "      if (msg) {\n"
    << "        float* wbuf = reinterpret_cast<float*>(smem + OFF_WB) + (threadIdx.x >> 5) * WB;\n"
    << "#pragma unroll\n        for (int m1 = 0; m1 < " << N1 << "; ++m1) wbuf[lane * " << N1 << " + m1] = mx[m1];\n"
    << "        __syncwarp();\n"
    << "        const int nch = min(32, " << MUL << " - u0 - r * 32);\n"
    << "        if (nch > 0) warp_copy_out(msg + (size_t)e * DIN + " << P.x_off[r.irrep] << " + (u0 + r * 32) * "
    << N1 << ", wbuf, nch * " << N1 << ", lane);\n"
    << "        __syncwarp();\n      }\n"
    << "      }\n";  // r
  if (combined) {
    o << "      if (sdy) {\n";
    for (int off = 0, rest = VZ; rest > 0;) {
      int V = 1;
      while (V * 2 <= rest && V * 2 <= 32) V *= 2;
      const int LV = __builtin_ctz(V), sh = 5 - LV;
      o << "        {\n          float zp[" << V << "];\n#pragma unroll\n          for (int t = 0; t < " << V
        << "; ++t) zp[t] = z[" << off << " + t];\n"
        << "          const float v = warp_sum_many<" << V << ">(zp, lane);\n"
        << "          if ((lane & " << ((1 << sh) - 1) << ") == 0) sdy[" << off << " + (lane >> " << sh
        << ")] = v;\n        }\n";
      off += V;
      rest -= V;
    }
    o << "      }\n";
  } else {
    for (int l2 = 0; l2 <= P.L; ++l2)
      if (!l2seen[l2])
        o << "      if (sdy && lane == 0) {\n#pragma unroll\n        for (int t = 0; t < " << 2 * l2 + 1
          << "; ++t) sdy[" << l2 * l2 << " + t] = 0.f;\n      }\n";
  }
  o << "    }\n    __syncwarp();\n    if (lane == 0) mbar_arrive(empty0 + 8 * s);\n  }\n"
    << "  __syncwarp();\n  if (lane == 0) mbar_arrive(gempty0 + 8 * gb);\n  ++kr;\n  }\n  *qp = q;\n  *kp = kr;\n}\n";
}

}  // namespace

static std::string gen_bwd_source(const Plan& P, const std::vector<SliceLayout>& SL, const KernelShape& K,
                                  const std::string& kname, int min_blocks) {
  const FwdConfig& F = P.bcfg;
  const int S = K.S, NW = K.nw;
  std::ostringstream o;
  o << spin_limit_define() << kPrelude;
  o << gen_common_device(P, SL, K, true);

  std::vector<int> slice_of(P.bwd_roles.size(), -1);
  for (int s = 0; s < S; ++s)
    for (int v : F.slice_roles[s]) slice_of[v] = s;
  std::vector<int> shape_of(P.bwd_roles.size(), -1), shape_rep;
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
  const std::string params =
      "(const int* __restrict__ rowptr, int n_recv, const int* __restrict__ eid, float* __restrict__ dW,\n"
      "    float* __restrict__ msg, int* __restrict__ err, unsigned char* smem, int u0, int ph, int nph, int chs,\n"
      "    bool want_dy, int* qp, int* kp)";
  for (size_t k = 0; k < shape_rep.size(); ++k) {
    const BwdRole& r = P.bwd_roles[shape_rep[k]];
    const SliceLayout& sl = SL[slice_of[shape_rep[k]]];
    if (K.no_chat) {
      gen_bwd_role_cg_first(o, P, K, r, sl, k, params);
      continue;
    }
    const Irrep& h = P.in[r.irrep];
    const int N1 = 2 * h.l + 1, R = r.R, MUL = h.mul;
    std::vector<int> ps;
    for (size_t q = 0; q < P.paths.size(); ++q)
      if (P.paths[q].irrep == r.irrep) ps.push_back((int)q);
    o << "// shape " << k << ": irrep " << r.irrep << " (" << h.mul << "x" << h.l << "), R=" << R << ", "
      << ps.size() << " paths\n";
    o << "__device__ __noinline__ void bcons_" << k << params << " {\n"
      << "  const int lane = threadIdx.x & 31;\n"
      << "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
      << "  const u32 gfull0 = full0 + OFF_GFULL, gempty0 = full0 + OFF_GEMPTY;\n"

      << "  int q = *qp, kr = *kp;\n"
      << "#pragma unroll 1\n  for (int i = RECV_FIRST; i < RECV_END; i += RECV_STEP) {\n"
      << "  const int e0 = EDGE_LO(i), e1 = EDGE_HI(i);\n"
      << "  if (e1 <= e0) continue;\n"
      << "  const int gb = kr % GBUF;\n"
      << "  if (!mbar_wait(gfull0 + 8 * gb, (kr / GBUF) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
      << "  const float* sg = reinterpret_cast<const float*>(smem + OFF_G) + gb * GS;\n"
      << "#pragma unroll 1\n  for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
      << "    const int s = q % NSTAGE;\n"
      << "    if (!stage_ready(full0, s, (q / NSTAGE) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
      << "    const int nb = min(NB, e1 - eb);\n"
      << "    unsigned char* st = stage_ptr(smem, s);\n"
      << "    const float* sW = reinterpret_cast<const float*>(st + OFF_W);\n"
      << "    const float* sX = reinterpret_cast<const float*>(st + OFF_X) + " << sl.x_st.at(r.irrep) << ";\n"
      << "    const float* sC = reinterpret_cast<const float*>(st + OFF_CH);\n"
      << "    float* sdyw = reinterpret_cast<float*>(st + OFF_DY) + (threadIdx.x >> 5) * NB * DE;\n"
      << "#pragma unroll 1\n    for (int b = ph; b < nb; b += nph) {\n"
      << "      const int e = eb + b;\n"
      << "      const float* wr = sW + b * WS;\n"
      << "      const float* xr = sX + b * XS;\n"
      << "      const float* chb = sC + b * chs;\n"
      << (K.tangent ? "      const float* chtb = reinterpret_cast<const float*>(st + OFF_CHT) + b * chs;\n"
                      "      const float* wtr = reinterpret_cast<const float*>(st + OFF_WT) + b * WS;\n"
                      "      const float* xtr = reinterpret_cast<const float*>(st + OFF_XT) + " +
                          std::to_string(sl.x_st.at(r.irrep)) + " + b * XS;\n"
                    : "")
      << "      float* dWrow = dW ? dW + (size_t)(eid ? __ldg(eid + e) : e) * NU : nullptr;\n"
      << "      float* sdy = want_dy ? sdyw + b * DE : nullptr;\n"
      ;
    // The R channel blocks of the role: RU of them unrolled together, the
    // groups of RU one after another in a loop.  Few channels per lane at a
    // time keep registers and code small; the Chat rows are read again per
    // group (broadcast loads).
    auto pow2 = [](int n) { int v = 1; while (v < n) v <<= 1; return v; };
    const bool combined = P.D_e <= 32;
    if (!combined && R != 1) {
      std::fprintf(stderr, "cgtp: backward role with R > 1 needs D_e <= 32\n");
      std::abort();
    }
    const int RU = bwd_unroll(N1, R);
    const int VZ = (int)P.D_e;  // reduced in power-of-two parts (9 = 8 + 1, 25 = 16 + 8 + 1)
    if (combined)
      o << "      float z[" << VZ << "];\n#pragma unroll\n      for (int t = 0; t < " << VZ << "; ++t) z[t] = 0.f;\n";
    o << "#pragma unroll 1\n      for (int r = 0; r < " << R << "; r += " << RU << ") {\n"
      << "      bool ok[" << RU << "];\n"
      << "      float xv[" << RU << "][" << N1 << "], mx[" << RU << "][" << N1 << "];\n"
      << (K.tangent ? "      float xtv[" + std::to_string(RU) + "][" + std::to_string(N1) + "];\n" : "")
      << "#pragma unroll\n      for (int v = 0; v < " << RU << "; ++v) {\n"
      << "        const int u = u0 + (r + v) * 32 + lane;\n"
      << "        ok[v] = " << (MUL % (32 * R) == 0 ? std::string("true") : "u < " + std::to_string(MUL))
      << ";  // every lane holds a channel when the blocks are full\n"
      << "#pragma unroll\n        for (int m1 = 0; m1 < " << N1
      << "; ++m1) { mx[v][m1] = 0.f; xv[v][m1] = ok[v] ? xr[u * " << N1 << " + m1] : 0.f; }\n";
    if (K.tangent)
      o << "#pragma unroll\n        for (int m1 = 0; m1 < " << N1 << "; ++m1) xtv[v][m1] = ok[v] ? xtr[u * " << N1
        << " + m1] : 0.f;\n";
    o << "      }\n";
    std::vector<char> l2seen(P.L + 1, 0);
    size_t q = 0;
    while (q < ps.size()) {
      const int l2 = P.paths[ps[q]].l2;
      const int N2 = 2 * l2 + 1;
      const int zo = combined ? l2 * l2 : 0;  // offset of degree l2 inside z
      l2seen[l2] = 1;
      o << "      {\n";
      if (!combined)
        o << "        float z[" << pow2(N2) << "];\n#pragma unroll\n        for (int t = 0; t < " << pow2(N2)
          << "; ++t) z[t] = 0.f;\n";
      for (; q < ps.size() && P.paths[ps[q]].l2 == l2; ++q) {
        const int pi = ps[q];
        const Path& p = P.paths[pi];
        const int N3 = 2 * p.l3 + 1, n2 = 2 * p.l2 + 1;
        o << "        {\n          float w[" << RU << "], gv[" << RU << "][" << N3 << "], dw[" << RU << "];\n"
          << (K.tangent ? "          float wt[" + std::to_string(RU) + "];\n" : "")
          << "#pragma unroll\n          for (int v = 0; v < " << RU << "; ++v) {\n"
          << "            const int u = u0 + (r + v) * 32 + lane;\n"
          << "            w[v] = ok[v] ? wr[" << sl.w_st.at(pi) << " + u] : 0.f;\n"
          << (K.tangent ? "            wt[v] = ok[v] ? wtr[" + std::to_string(sl.w_st.at(pi)) + " + u] : 0.f;\n" : "")
          << "#pragma unroll\n            for (int m3 = 0; m3 < " << N3 << "; ++m3) gv[v][m3] = ok[v] ? sg["
          << sl.g_st.at(pi) << " + u * " << N3 << " + m3] : 0.f;\n          }\n";
        if (K.tangent)
          o << "          bpath_tan<" << N1 << "," << N3 << "," << RU << ">(chb + " << sl.ch_off.at(pi) << ", chtb + "
            << sl.ch_off.at(pi) << ", xv, xtv, w, wt, gv, mx, dw);\n";
        else
          o << "          bpath<" << N1 << "," << N3 << "," << RU << ">(chb + " << sl.ch_off.at(pi)
            << ", xv, w, gv, mx, dw);\n";
        o
          << "          if (dWrow) {\n#pragma unroll\n            for (int v = 0; v < " << RU
          << "; ++v) if (ok[v]) dWrow[" << p.k0 << " + u0 + (r + v) * 32 + lane] = dw[v];\n          }\n"
          << "          if (sdy) {\n#pragma unroll\n            for (int v = 0; v < " << RU << "; ++v) {\n"
          << "              float wx[" << N1 << "];\n#pragma unroll\n              for (int m1 = 0; m1 < " << N1
          << (K.tangent ? "; ++m1) wx[m1] = fmaf(w[v], xtv[v][m1], wt[v] * xv[v][m1]);  // d (w x)\n"
                        : "; ++m1) wx[m1] = w[v] * xv[v][m1];\n");
        const double* C = P.coeff.data() + p.c_off;
        for (int m1 = 0; m1 < N1; ++m1)
          for (int m3 = 0; m3 < N3; ++m3) {
            std::vector<std::pair<int, double>> t;
            for (int m2 = 0; m2 < n2; ++m2) {
              const double c = C[((size_t)m1 * n2 + m2) * N3 + m3];
              if (c != 0.0) t.push_back({m2, c});
            }
            if (t.empty()) continue;
            o << "              { const float pr = wx[" << m1 << "] * gv[v][" << m3 << "];";
            for (auto& tc : t)
              o << " z[" << zo + tc.first << "] = fmaf(" << flt(tc.second) << ", pr, z[" << zo + tc.first << "]);";
            o << " }\n";
          }
        o << "            }\n          }\n        }\n";
      }
      if (!combined) {
        const int V = pow2(N2), LV = __builtin_ctz(V), sh = 5 - LV;
        o << "        if (sdy) {\n          const float v = warp_sum_many<" << V << ">(z, lane);\n"
          << "          const int k = lane >> " << sh << ";\n"
          << "          if ((lane & " << ((1 << sh) - 1) << ") == 0 && k < " << N2 << ") sdy[" << l2 * l2
          << " + k] = v;\n        }\n";
      }
      o << "      }\n";
    }
    // this group's message row segment, through the warp's buffer
    o << "      if (msg) {\n"
      << "        float* wbuf = reinterpret_cast<float*>(smem + OFF_WB) + (threadIdx.x >> 5) * WB;\n"
      << "#pragma unroll\n        for (int v = 0; v < " << RU << "; ++v) {\n"
      << "#pragma unroll\n          for (int m1 = 0; m1 < " << N1 << "; ++m1) wbuf[(v * 32 + lane) * " << N1
      << " + m1] = mx[v][m1];\n        }\n"
      << "        __syncwarp();\n"
      << "        const int nch = min(" << 32 * RU << ", " << MUL << " - u0 - r * 32);\n"
      << "        if (nch > 0) warp_copy_out(msg + (size_t)e * DIN + " << P.x_off[r.irrep] << " + (u0 + r * 32) * "
      << N1 << ", wbuf, nch * " << N1 << ", lane);\n"
      << "        __syncwarp();\n      }\n"
      << "      }\n";  // r
    if (combined) {
      o << "      if (sdy) {\n";
      for (int off = 0, rest = VZ; rest > 0;) {
        int V = 1;
        while (V * 2 <= rest && V * 2 <= 32) V *= 2;
        const int LV = __builtin_ctz(V), sh = 5 - LV;
        o << "        {\n          float zp[" << V << "];\n#pragma unroll\n          for (int t = 0; t < " << V
          << "; ++t) zp[t] = z[" << off << " + t];\n"
          << "          const float v = warp_sum_many<" << V << ">(zp, lane);\n"
          << "          if ((lane & " << ((1 << sh) - 1) << ") == 0) sdy[" << off << " + (lane >> " << sh
          << ")] = v;\n        }\n";
        off += V;
        rest -= V;
      }
      o << "      }\n";
    } else {
      for (int l2 = 0; l2 <= P.L; ++l2)
        if (!l2seen[l2])
          o << "      if (sdy && lane == 0) {\n#pragma unroll\n        for (int t = 0; t < " << 2 * l2 + 1
            << "; ++t) sdy[" << l2 * l2 << " + t] = 0.f;\n      }\n";
    }
    o << "    }\n    __syncwarp();\n    if (lane == 0) mbar_arrive(empty0 + 8 * s);\n  }\n"
      << "  __syncwarp();\n  if (lane == 0) mbar_arrive(gempty0 + 8 * gb);\n  ++kr;\n  }\n  *qp = q;\n  *kp = kr;\n}\n";
  }
  o << "__device__ __noinline__ void bcons_idle" << params << " {\n"
       "  const int lane = threadIdx.x & 31;\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  const u32 gempty0 = full0 + OFF_GEMPTY;\n"
       "  int q = *qp, kr = *kp;\n"
       "#pragma unroll 1\n  for (int i = RECV_FIRST; i < RECV_END; i += RECV_STEP) {\n"
       "    const int e0 = EDGE_LO(i), e1 = EDGE_HI(i);\n"
       "    if (e1 <= e0) continue;\n"
       "    for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
       "      const int s = q % NSTAGE;\n"
       "      if (!stage_ready(full0, s, (q / NSTAGE) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
       "      __syncwarp();\n"
       "      if (lane == 0) mbar_arrive(empty0 + 8 * s);\n"
       "    }\n"
       "    if (lane == 0) mbar_arrive(gempty0 + 8 * (kr % GBUF));\n"
       "    ++kr;\n"
       "  }\n"
       "  *qp = q;\n"
       "  *kp = kr;\n"
       "}\n";
  o << "__constant__ int kShape[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? shape_of[F.slice_roles[s][w]] : -1) << ",";
  o << "};\n__constant__ int kU0[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? P.bwd_roles[F.slice_roles[s][w]].u0 : 0) << ",";
  o << "};\n__constant__ int kEntBegin[" << S + 1 << "] = {";
  for (int v : P.bwd_ent_begin) o << v << ",";
  o << "};\n";
  o << "extern \"C\" __global__ void __launch_bounds__((NW + 2) * 32, " << min_blocks << ") " << kname
    << "(const int* __restrict__ rowptr, const int* __restrict__ col, const float* __restrict__ x,\n"
       "    const float* __restrict__ Y, const float* __restrict__ W, const int* __restrict__ eid,\n"
       "    const float* __restrict__ g, float* __restrict__ dW, float* __restrict__ dyp, float* __restrict__ msg,\n"
       "    const int4* __restrict__ ent, int n_recv, int* __restrict__ err, int e_stride"
    << (K.tangent ? ",\n    const float* __restrict__ xt, const float* __restrict__ Yt, const float* __restrict__ Wt"
                  : "")
    << ") {\n"
       "  extern __shared__ __align__(128) unsigned char smem[];\n"
       "  grid_dependency_wait();  // the previous kernel's results are visible\n"
       "  grid_launch_dependents();\n"
       "  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  const u32 gfull0 = full0 + OFF_GFULL, gempty0 = full0 + OFF_GEMPTY;\n"
       "  if (threadIdx.x == 0) {\n"
       "    for (int s = 0; s < NSTAGE; ++s) {\n"
       "      mbar_init(full0 + 8 * s, FULL_COUNT); mbar_init(empty0 + 8 * s, NW); mbar_init(full0 + OFF_CHAT + 8 * s, CHAT_COUNT);\n"
       "    }\n"
       "    for (int b = 0; b < 2; ++b) { mbar_init(gfull0 + 8 * b, 32); mbar_init(gempty0 + 8 * b, NW); }\n"
       "    fence_mbar_init();\n"
       "  }\n"
       << (K.edge_ranges
           ? "  if (warp == 0) {  // this CTA's share of the edges and the receivers it touches\n"
             "    const int E = __ldg(rowptr + n_recv);\n"
             "    const int lo = (int)((long long)E * blockIdx.x / gridDim.x);\n"
             "    const int hi = (int)((long long)E * (blockIdx.x + 1) / gridDim.x);\n"
             "    const int i0 = warp_last_le(rowptr, 0, n_recv - 1, lo, lane);\n"
             "    const int i1 = hi > lo ? warp_last_le(rowptr, 0, n_recv - 1, hi - 1, lane) + 1 : i0;\n"
             "    if (lane == 0) *reinterpret_cast<int4*>(smem + OFF_RANGE) = make_int4(i0, i1, lo, hi);\n"
             "  }\n"
           : "") <<
       "  __syncthreads();\n"
    << (K.tangent ? "" : "  const float* xt = nullptr; const float* Yt = nullptr; const float* Wt = nullptr;\n")
    << "  if (warp == NW) { tma_warp(rowptr, n_recv, col, x, W, xt, Wt, eid, g, err, smem, lane); return; }\n"
       "  if (warp == NW + 1) { helper_warp(rowptr, n_recv, Y, Yt, ent, kEntBegin, dyp, err, smem, lane, e_stride); return; }\n"
       "  int q = 0, kr = 0;\n"
       "  for (int slice = 0; slice < NSLICE; ++slice) {\n"
       "    const int slot = slice * NW + warp;\n"
       "    const int u0 = kU0[slot], ph = kPh[slot], nph = kNph[slot], chs = kChs[slice];\n"
       "    switch (kShape[slot]) {\n";
  for (size_t k = 0; k < shape_rep.size(); ++k)
    o << "    case " << k << ": bcons_" << k
      << "(rowptr, n_recv, eid, dW, msg, err, smem, u0, ph, nph, chs, dyp != nullptr, &q, &kr); break;\n";
  o << "    default: bcons_idle(rowptr, n_recv, eid, dW, msg, err, smem, u0, ph, nph, chs, dyp != nullptr, &q, &kr); break;\n"
       "    }\n"
       "    if (q < 0) break;  // a wait expired: this warp stops\n  }\n}\n";
  return o.str();
}

namespace {

// One backward warp role option for a hidden irrep: R channels per lane,
// nph edge phases.
struct BwdOption {
  int R, nph, roles;
  double cost;  // instructions per chunk of the costliest role
};

struct BwdIrrep {
  int a;
  std::vector<BwdOption> opts;
};

// Instructions one warp issues per edge for R channel sets of irrep a (all
// its paths): the s, dW, msg and dY arithmetic, shared loads, stores, and the
// lane reduction of the dY partials.
double bwd_edge_cost(const Plan& P, int a, int R) {
  const int n1 = 2 * P.in[a].l + 1;
  auto pow2 = [](int n) { int v = 1; while (v < n) v <<= 1; return v; };
  double c = 2.0 * R * n1 + 12.0 * ((R + bwd_unroll(n1, R) - 1) / bwd_unroll(n1, R));  // x, msg, loop
  std::vector<char> l2seen(P.L + 1, 0);
  for (size_t k = 0; k < P.paths.size(); ++k) {
    const Path& p = P.paths[k];
    if (p.irrep != a) continue;
    const int n2 = 2 * p.l2 + 1, n3 = 2 * p.l3 + 1;
    int nnz = 0, pairs = 0;
    const double* C = P.coeff.data() + p.c_off;
    for (int m1 = 0; m1 < n1; ++m1)
      for (int m3 = 0; m3 < n3; ++m3) {
        int t = 0;
        for (int m2 = 0; m2 < n2; ++m2) t += C[((size_t)m1 * n2 + m2) * n3 + m3] != 0.0;
        nnz += t;
        pairs += t > 0;
      }
    const int groups = (R + bwd_unroll(n1, R) - 1) / bwd_unroll(n1, R);
    c += R * ((double)n1 * n3 + 3.0 * n1 + n3 + 2.0 + pairs + nnz) + groups * (double)n3 * ((n1 + 3) / 4);
    l2seen[p.l2] = 1;
  }
  if (P.D_e <= 32) {
    c += 2.0 * pow2((int)P.D_e) + 8.0;
  } else {
    for (int l2 = 0; l2 <= P.L; ++l2)
      if (l2seen[l2]) c += 2.0 * pow2(2 * l2 + 1) + 8.0;
  }
  return c;
}

// Registers per thread the compiler grants a block of `threads` threads when
// `ctas` blocks share an SM: each of the four schedulers has 16384 registers
// for its share of the warps (rounded up), in eight-register steps.
int reg_cap(int threads, int ctas) {
  const int warps_per_sched = ((threads / 32) * ctas + 3) / 4;
  return std::min(255, 16384 / (warps_per_sched * 32) / 8 * 8);
}

// Registers a backward role of irrep a with R channels per lane keeps live:
// the dY partials, x, msg and s per channel, grad_out of the widest path, the
// Chat row, and about 28 for addresses, counters and temporaries.
int bwd_role_regs(const Plan& P, int a, int R) {
  const int n1 = 2 * P.in[a].l + 1;
  int n3max = 1;
  for (auto& p : P.paths)
    if (p.irrep == a) n3max = std::max(n3max, 2 * p.l3 + 1);
  auto pow2 = [](int n) { int v = 1; while (v < n) v <<= 1; return v; };
  int vz = 0;
  if (P.D_e <= 32) {
    vz = pow2((int)P.D_e);
  } else {
    for (auto& p : P.paths)
      if (p.irrep == a) vz = std::max(vz, pow2(2 * p.l2 + 1));
  }
  // a tenth on top: the compiler keeps a few more values live than these
  const int RU = bwd_unroll(n1, R);  // blocks unrolled together; the rest loop
  return (28 + vz + RU * (3 * n1 + n3max + 2) + n1 + ((n1 + 3) & ~3)) * 11 / 10;
}

// Smallest per-chunk time of a slice holding the given irreps with NW warps:
// the least bound T such that every irrep has an option no costlier than T
// and the options' roles fit NW.  Returns -1 when nothing fits.
double slice_time(const std::vector<BwdIrrep>& W, const std::vector<int>& members, int NW,
                  std::vector<int>* choice) {
  std::vector<double> cand;
  for (int m : members)
    for (auto& o : W[m].opts) cand.push_back(o.cost);
  std::sort(cand.begin(), cand.end());
  cand.erase(std::unique(cand.begin(), cand.end()), cand.end());
  for (double T : cand) {
    int roles = 0;
    std::vector<int> pick;
    bool ok = true;
    for (int m : members) {
      int best = -1;
      for (size_t k = 0; k < W[m].opts.size(); ++k) {
        const BwdOption& o = W[m].opts[k];
        if (o.cost <= T && (best < 0 || o.roles < W[m].opts[best].roles ||
                            (o.roles == W[m].opts[best].roles && o.cost < W[m].opts[best].cost)))
          best = (int)k;
      }
      if (best < 0) {
        ok = false;
        break;
      }
      roles += W[m].opts[best].roles;
      pick.push_back(best);
    }
    if (ok && roles <= NW) {
      if (choice) *choice = pick;
      return T;
    }
  }
  return -1.0;
}

// Every set partition of {0..n-1} as restricted growth strings.
void partitions(int n, std::vector<std::vector<int>>& out) {
  std::vector<int> a(n, 0);
  std::function<void(int, int)> rec = [&](int i, int mx) {
    if (i == n) {
      out.push_back(a);
      return;
    }
    for (int v = 0; v <= mx + 1; ++v) {
      a[i] = v;
      rec(i + 1, std::max(mx, v));
    }
  };
  if (n > 0) rec(0, -1);
}

}  // namespace

cgtp_status build_backward(Plan& P) {
  P.bwd_roles.clear();
  FwdConfig& F = P.bcfg;
  F = FwdConfig();
  if (P.paths.empty()) return CGTP_OK;
  // ---- per hidden irrep: the edge cost of each channel width per lane
  std::vector<int> work_irreps;
  for (size_t a = 0; a < P.in.size(); ++a) {
    bool any = false;
    for (auto& p : P.paths) any = any || p.irrep == (int)a;
    if (any)
      work_irreps.push_back((int)a);
    else
      P.bwd_irrep_gap = true;
  }
  const int n = (int)work_irreps.size();
  std::vector<std::vector<int>> parts;
  if (n <= 8) {
    partitions(n, parts);
  } else {  // one slice per irrep
    std::vector<int> a(n);
    std::iota(a.begin(), a.end(), 0);
    parts.push_back(a);
  }
  struct Best {
    double score = 1e300;
    int B = 0, NW = 0, ctas = 0;
    std::vector<std::vector<int>> slices;  // members (indices into work_irreps)
    std::vector<std::vector<int>> pick;    // option per member
    std::vector<BwdIrrep> W;
  } best;
  // Candidates (chunk, least resident CTAs per SM) in order of preference,
  // from measurements on B200: the largest chunk of at least four edges that
  // leaves two CTAs per SM (the chunk sets how many edges each stage hands
  // over per barrier round trip, and how many are in flight); when none
  // does, four edges at one CTA (wide rows: Lmax 2 wide 297 -> 270 us, Lmax 6
  // 2130 -> 1917 us against eight edges at one CTA), then smaller chunks.
  // Among the plans of a candidate: the shortest consumer critical path per
  // SM.
  std::vector<std::pair<int, int>> cand = {{8, 2}, {4, 2}, {4, 1}, {2, 1}, {1, 1}};
  if (const char* v = std::getenv("CGTP_BWD_CHUNK")) {  // tuning override: one chunk size
    const int B0 = std::max(1, std::min(8, std::atoi(v)));
    cand = {{B0, 2}, {B0, 1}};
  }
  // barrier round trips, loop and address work of one chunk, in the units of
  // bwd_edge_cost
  const double kChunkOverhead = 80.0;
  // consumer warps per CTA: 6, 12 and 16 measured slower than 4 or 8 on B200
  int kNW[] = {4, 8};
  if (const char* v = std::getenv("CGTP_BWD_NW"))  // tuning override: one warp count
    kNW[0] = kNW[1] = std::max(1, std::min(16, std::atoi(v)));
  for (const auto& [B, min_ctas] : cand) {
    if (best.B != 0) break;
    // options of every irrep for this chunk size
    std::vector<BwdIrrep> W(n);
    for (int i = 0; i < n; ++i) {
      const int a = work_irreps[i];
      const Irrep& h = P.in[a];
      W[i].a = a;
      // channel blocks one warp takes in turn (the dY partials of all blocks
      // must fit one reduction: only when (L+1)^2 <= 32)
      std::vector<int> Rs = {1};
      if (P.D_e <= 32) {
        if (h.mul > 32) Rs.push_back(2);
        if (h.mul > 64) Rs.push_back(4);
      }
      for (int R : Rs) {
        const double ce = bwd_edge_cost(P, a, R);
        const int nblk = (h.mul + 32 * R - 1) / (32 * R);
        for (int nph = 1; nph <= B; nph *= 2)
          W[i].opts.push_back({R, nph, nblk * nph, ce * ((B + nph - 1) / nph)});
      }
    }
    for (int NW : kNW) {
      for (const auto& rgs : parts) {
        const int ns = rgs.empty() ? 0 : *std::max_element(rgs.begin(), rgs.end()) + 1;
        std::vector<std::vector<int>> slices(ns);
        for (int i = 0; i < n; ++i) slices[rgs[i]].push_back(i);
        double sumT = 0.0;
        std::vector<std::vector<int>> pick(ns);
        bool ok = true;
        for (int s2 = 0; s2 < ns && ok; ++s2) {
          const double T = slice_time(W, slices[s2], NW, &pick[s2]);
          if (T < 0) ok = false;
          sumT += T + kChunkOverhead;
        }
        if (!ok) continue;
        // shared memory of this grouping at this chunk size
        std::vector<SliceLayout> SL(ns);
        KernelShape K;
        K.S = ns;
        K.nw = NW;
        K.force_B = B;
        K.no_chat = P.bwd_tform;
        int maxr = 0;
        for (int s2 = 0; s2 < ns; ++s2) {
          for (size_t k = 0; k < slices[s2].size(); ++k) {
            const int a = W[slices[s2][k]].a;
            const BwdOption& o = W[slices[s2][k]].opts[pick[s2][k]];
            SL[s2].irreps.push_back(a);
            for (size_t q = 0; q < P.paths.size(); ++q)
              if (P.paths[q].irrep == a) SL[s2].paths.push_back((int)q);
            K.WB = std::max(K.WB, 32 * bwd_unroll(2 * P.in[a].l + 1, o.R) * (2 * P.in[a].l + 1));
            maxr = std::max(maxr, bwd_role_regs(P, a, o.R));
          }
          std::sort(SL[s2].paths.begin(), SL[s2].paths.end());
          layout_slice(P, SL[s2], true);
        }
        plan_layout(P, SL, K, true);
        if (K.smem > 227 * 1024) continue;
        // resident CTAs: shared memory, warps, and a register estimate
        // the most CTAs (up to three) whose register share still holds the
        // role's estimate; none: the roles would spill
        const int threads = (NW + 2) * 32;
        int ctas = 0;
        for (int c = std::min({3, 233472 / (K.smem + 1024), 64 / (NW + 2)}); c >= 1 && !ctas; --c)
          if (maxr <= reg_cap(threads, c)) ctas = c;
        if (ctas < min_ctas) continue;
        // resident CTAs weigh more than their count: each brings its own ring
        // of stages, so the SM keeps more loads in flight
        const double score = sumT / std::pow((double)ctas, 1.5) * (1.0 + 0.01 * NW);
        if (score < best.score) {
          best.score = score;
          best.B = B;
          best.NW = NW;
          best.slices = slices;
          best.pick = pick;
          best.W = W;
          best.ctas = ctas;
        }
      }
    }
  }
  if (best.B == 0) return fail(CGTP_ERR_SIZE, "backward kernel needs too much shared memory");
  // ---- roles of the chosen plan: channel blocks x edge phases per irrep
  F.S = (int)best.slices.size();
  F.nw = best.NW;
  F.slice_roles.assign(F.S, {});
  std::vector<SliceLayout> SL(F.S);
  KernelShape K;
  K.S = F.S;
  K.nw = F.nw;
  K.force_B = best.B;
  K.no_chat = P.bwd_tform;
  for (int s2 = 0; s2 < F.S; ++s2) {
    for (size_t k = 0; k < best.slices[s2].size(); ++k) {
      const BwdIrrep& wi = best.W[best.slices[s2][k]];
      const BwdOption& o = wi.opts[best.pick[s2][k]];
      const Irrep& h = P.in[wi.a];
      const int nblk = (h.mul + 32 * o.R - 1) / (32 * o.R);
      for (int blk = 0; blk < nblk; ++blk)
        for (int ph = 0; ph < o.nph; ++ph) {
          BwdRole r;
          r.irrep = wi.a;
          r.u0 = blk * 32 * o.R;
          r.R = o.R;
          r.ph = ph;
          r.nph = o.nph;
          r.cost = o.cost;
          F.slice_roles[s2].push_back((int)P.bwd_roles.size());
          P.bwd_roles.push_back(r);
        }
      SL[s2].irreps.push_back(wi.a);
      for (size_t q = 0; q < P.paths.size(); ++q)
        if (P.paths[q].irrep == wi.a) SL[s2].paths.push_back((int)q);
      K.WB = std::max(K.WB, 32 * bwd_unroll(2 * h.l + 1, o.R) * (2 * h.l + 1));
    }
    std::sort(SL[s2].paths.begin(), SL[s2].paths.end());
    layout_slice(P, SL[s2], true);
  }
  plan_layout(P, SL, K, true);
  F.B = K.B;
  F.stages = K.stages;
  F.w_smem = K.w_bulk;
  F.x_smem = K.x_bulk;

  cgtp_status st = upload_chat_tables(P, SL, &P.d_bwd_ent, P.bwd_ent_begin);
  if (st != CGTP_OK) return st;
  for (size_t k = 0; k + 1 < P.bwd_ent_begin.size(); ++k)
    K.rec_max = std::max(K.rec_max, P.bwd_ent_begin[k + 1] - P.bwd_ent_begin[k]);
  // register cap from the resident CTAs shared memory allows; one CTA fewer
  // (but not below two) when the compiler reports sizeable spills
  if (K.smem > 227 * 1024) return fail(CGTP_ERR_SIZE, "backward kernel needs too much shared memory");
  bool fixed = false;
  int mb0 = initial_min_blocks(K.smem, &fixed);
  if (!fixed) mb0 = std::min(mb0, best.ctas);  // the planner's register share
  if (const char* v = std::getenv("CGTP_BWD_MIN_BLOCKS")) {
    mb0 = std::max(1, std::atoi(v));
    fixed = true;
  }
  const int mb_floor = fixed ? mb0 : std::min(mb0, 2);
  // Two variants of the same kernel: CTAs over whole receivers, and CTAs
  // over equal edge ranges.  The second balances graphs with few receivers
  // per CTA; measured on B200, the range code in the first variant (even
  // when not taken) slowed the large cases, hence two kernels.
  // Both are compiled at once on two host threads (NVRTC needs no CUDA
  // context; each takes tens of seconds at Lmax 6), then loaded here.  Each
  // lowers its resident-CTA target while the compiler reports spills.
  struct Variant {
    std::string src;
    JitBinary bin;
    cgtp_status st = CGTP_OK;
  } var[2];
  auto build = [&](int er) {
    try {
      KernelShape Kv = K;
      Kv.edge_ranges = er == 1;
      const std::string name = er ? "cgtp_bwd_er" : "cgtp_bwd";
      for (int mb = mb0; mb >= mb_floor; --mb) {
        var[er].src = gen_bwd_source(P, SL, Kv, name, mb);
        var[er].st = jit_build(var[er].src, name, var[er].bin);
        if (var[er].st != CGTP_OK || mb == mb_floor || max_spill_bytes(var[er].bin.log) <= 160) break;
      }
    } catch (const std::exception& e) {
      var[er].st = CGTP_ERR_OOM;
      var[er].bin.err = std::string("exception while building the backward: ") + e.what();
    }
  };
  {
    std::thread second;
    try {
      second = std::thread(build, 1);
    } catch (...) {
    }
    build(0);
    if (second.joinable())
      second.join();
    else
      build(1);
  }
  for (int er = 0; er < 2; ++er) {
    if (var[er].st != CGTP_OK) {
      set_error(var[er].bin.err);
      return var[er].st;
    }
    JitKernel& JK = er ? P.bwd_er : P.bwd;
    JK.threads = (F.nw + 2) * 32;
    JK.smem = K.smem;
    cgtp_status cst = jit_load(var[er].bin, er ? "cgtp_bwd_er" : "cgtp_bwd", JK);
    if (cst != CGTP_OK) return cst;
    if (const char* d = std::getenv("CGTP_DUMP_SOURCE")) {
      FILE* f = std::fopen((std::string(d) + (er ? "/bwd_er.cu" : "/bwd.cu")).c_str(), "w");
      if (f) {
        std::fputs(var[er].src.c_str(), f);
        std::fclose(f);
      }
    }
  }
  return CGTP_OK;
}

// The backward's tangent kernel (cgtp_bwd_tan): the same roles and slices
// as cgtp_bwd, every W, x and Y piece staged with its directional
// derivative, so that one pass gives d/dt of (dW, dY, the dx messages) at
// (x + t xt, Y + t Yt, W + t Wt) for a fixed grad_out.  The chunk is halved
// while the doubled stages do not fit.  Built on first use.
cgtp_status build_backward_tangent(Plan& P, JitKernel& out, std::string* src_out) {
  const FwdConfig& F = P.bcfg;
  std::vector<SliceLayout> SL(F.S);
  KernelShape K;
  K.S = F.S;
  K.nw = F.nw;
  K.tangent = true;
  K.no_chat = P.bwd_tform;
    for (int s2 = 0; s2 < F.S; ++s2) {
    for (int ri : F.slice_roles[s2]) {
      const BwdRole& r = P.bwd_roles[ri];
      auto& irr = SL[s2].irreps;
      if (std::find(irr.begin(), irr.end(), r.irrep) == irr.end()) {
        irr.push_back(r.irrep);
        for (size_t q = 0; q < P.paths.size(); ++q)
          if (P.paths[q].irrep == r.irrep) SL[s2].paths.push_back((int)q);
      }
      K.WB = std::max(K.WB, 32 * bwd_unroll(2 * P.in[r.irrep].l + 1, r.R) * (2 * P.in[r.irrep].l + 1));
    }
    std::sort(SL[s2].paths.begin(), SL[s2].paths.end());
    layout_slice(P, SL[s2], true);
  }
  // the largest chunk (at most the plain kernel's) whose doubled stages
  // leave room for two CTAs per SM; else the largest that fits one.  Never
  // below the roles' edge phases: a role takes the edges b of a chunk with
  // b % nph == ph, so a chunk of fewer than nph edges would leave the roles
  // of the higher phases without work.
  int min_B = 1;
  for (const BwdRole& r : P.bwd_roles) min_B = std::max(min_B, r.nph);
  int pick = 0;
  for (int B = F.B; B >= min_B && !pick; B /= 2) {
    K.force_B = B;
    plan_layout(P, SL, K, true);
    if (2 * (K.smem + 1024) <= 228 * 1024) pick = B;
  }
  for (int B = F.B; B >= min_B && !pick; B /= 2) {
    K.force_B = B;
    plan_layout(P, SL, K, true);
    if (K.smem <= 227 * 1024) pick = B;
  }
  if (!pick) return fail(CGTP_ERR_SIZE, "tangent backward needs too much shared memory");
  K.force_B = pick;
  plan_layout(P, SL, K, true);
  for (size_t k = 0; k + 1 < P.bwd_ent_begin.size(); ++k)
    K.rec_max = std::max(K.rec_max, P.bwd_ent_begin[k + 1] - P.bwd_ent_begin[k]);
  bool fixed = false;
  const int mb0 = initial_min_blocks(K.smem, &fixed);
  const int mb_floor = fixed ? mb0 : 1;  // down to one CTA while the doubled roles spill
  const std::string name = "cgtp_bwd_tan";
  std::string src;
  JitBinary bin;
  cgtp_status st = CGTP_OK;
  for (int mb = mb0; mb >= mb_floor; --mb) {
    src = gen_bwd_source(P, SL, K, name, mb);
    st = jit_build(src, name, bin);
    if (st != CGTP_OK || mb == mb_floor || max_spill_bytes(bin.log) <= 160) break;
  }
  if (st != CGTP_OK) {
    set_error(bin.err);
    return st;
  }
  out.threads = (F.nw + 2) * 32;
  out.smem = K.smem;
  if (src_out) *src_out = src;
  return jit_load(bin, name, out);
}

}  // namespace cgtp
