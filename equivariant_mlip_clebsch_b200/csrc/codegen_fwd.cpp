// codegen_fwd.cpp -- the forward CGTP convolution kernel, generated per plan.
//
// Node-centric execution (LunaTP Fig. 3a: every receiver's row is
// accumulated on chip and stored once, no atomics).  Persistent CTAs walk the
// slices of the warp roles in turn and, in each, the receivers blockIdx.x,
// + gridDim.x, ...  The TMA warp and the helper warp (codegen_common.cpp)
// stream a receiver's edges in chunks of NB through a ring of NSTAGE stages
// holding, per edge, the W and x pieces of the slice, the Y row and
// Chat = C.Y for the slice's paths.  Each consumer warp runs one role: R
// channels per lane of one hidden irrep and a group of that irrep's paths,
// accumulating
//     acc[p][u][m3] += W[e][k0_p+u] * sum_m1 Chat[m3][m1] x[j][u][m1]
// in registers.  x is read once per edge for all paths of the group (the
// cross-path input reuse of LunaTP Table 8); the paths of an irrep are
// grouped under a register budget per lane (LunaTP's output-component budget,
// Fig. 3b / Table 7).  Roles with the same irrep and path group share one
// __noinline__ function with the channel block as an argument.  Wide plans
// use one-path roles instead, one function per (2l1+1, 2l3+1) shape.  Plans
// with a hidden irrep of l >= 3 use packed roles (fpath2: float2 accumulators
// of m3 pairs over an m1-major Chat, one packed FMA per m1 and pair).  Two
// more kernels come from the same generator for the double backward: the
// tangent forward (every staged piece doubled) and the accumulating forward,
// which adds its rows to the output with red.global.add (one add per element
// per launch, so still deterministic).
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <memory>
#include <numeric>
#include <sstream>
#include <thread>
#include <tuple>

#include "codegen_common.hpp"

namespace cgtp {

// The kernel entry after the role functions: service warps, then each
// consumer warp runs its slot's role in every slice.
static void gen_fwd_entry(std::ostringstream& o, const std::string& kname, int min_blocks,
                          const std::string& dispatch, bool tangent) {
  o << "extern \"C\" __global__ void __launch_bounds__((NW + 2) * 32, " << min_blocks << ") " << kname
    << "(const int* __restrict__ rowptr, const int* __restrict__ col, const float* __restrict__ x,\n"
       "    const float* __restrict__ Y, const float* __restrict__ W, const int* __restrict__ eid,\n"
       "    float* __restrict__ out, const int4* __restrict__ ent, int n_recv, int* __restrict__ err"
    << (tangent ? ",\n    const float* __restrict__ xt, const float* __restrict__ Yt, const float* __restrict__ Wt"
                : "")
    << ") {\n"
       "  extern __shared__ __align__(128) unsigned char smem[];\n"
       "  grid_dependency_wait();  // the previous kernel's results are visible\n"
       "  grid_launch_dependents();\n"
       "  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  if (threadIdx.x == 0) {\n"
       "    for (int s = 0; s < NSTAGE; ++s) {\n"
       "      mbar_init(full0 + 8 * s, FULL_COUNT); mbar_init(empty0 + 8 * s, NW); mbar_init(full0 + OFF_CHAT + 8 * s, CHAT_COUNT);\n"
       "    }\n"
       "    fence_mbar_init();\n"
       "  }\n"
       "  __syncthreads();\n"
    << (tangent ? "" : "  const float* xt = nullptr; const float* Yt = nullptr; const float* Wt = nullptr;\n")
    << "  if (warp == NW) { tma_warp(rowptr, n_recv, col, x, W, xt, Wt, eid, nullptr, err, smem, lane); return; }\n"
       "  if (warp == NW + 1) { helper_warp(rowptr, n_recv, Y, Yt, ent, kEntBegin, nullptr, err, smem, lane, 0); return; }\n"
       "  int q = 0;\n"
       "  for (int slice = 0; slice < NSLICE; ++slice) {\n"
       "    const int slot = slice * NW + warp;\n"
       "    const int u0 = kU0[slot], chs = kChs[slice];\n"
       "    switch (kShape[slot]) {\n"
    << dispatch << "    default: fcons_idle(rowptr, n_recv, err, smem, &q); break;\n    }\n"
       "    if (q < 0) break;  // a wait expired: this warp stops\n  }\n}\n";
}

static void gen_fwd_idle(std::ostringstream& o) {
  // idle consumer: keeps the stage accounting of the CTA
  o << "__device__ __noinline__ void fcons_idle(const int* __restrict__ rowptr, int n_recv,\n"
       "    int* __restrict__ err, unsigned char* smem, int* qp) {\n"
       "  const int lane = threadIdx.x & 31;\n"
       "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
       "  int q = *qp;\n"
       "#pragma unroll 1\n  for (int i = RECV_FIRST; i < RECV_END; i += RECV_STEP) {\n"
       "    const int e0 = EDGE_LO(i), e1 = EDGE_HI(i);\n"
       "    for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
       "      const int s = q % NSTAGE;\n"
       "      if (!stage_ready(full0, s, (q / NSTAGE) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
       "      __syncwarp();\n"
       "      if (lane == 0) mbar_arrive(empty0 + 8 * s);\n"
       "    }\n"
       "  }\n"
       "  *qp = q;\n"
       "}\n";
}

// Wide plans: one function per (2l1+1, 2l3+1, full channel blocks) shape; a
// role's path offsets come from per-slot tables.
static std::string gen_fwd_generic(const Plan& P, const std::vector<SliceLayout>& SL, const KernelShape& K,
                                   const std::string& kname, int min_blocks, std::ostringstream& o,
                                   const std::vector<int>& slice_of) {
  const FwdConfig& F = P.fcfg;
  const int S = K.S, NW = K.nw;
  std::vector<std::tuple<int, int, bool>> shapes;
  std::vector<int> shape_of(P.fwd_roles.size(), -1);
  for (size_t ri = 0; ri < P.fwd_roles.size(); ++ri) {
    const FwdRole& r = P.fwd_roles[ri];
    const Path& p = P.paths[r.paths[0]];
    const auto key = std::make_tuple(2 * P.in[r.irrep].l + 1, 2 * p.l3 + 1, P.in[r.irrep].mul % 32 == 0);
    auto it = std::find(shapes.begin(), shapes.end(), key);
    shape_of[ri] = (int)(it - shapes.begin());
    if (it == shapes.end()) shapes.push_back(key);
  }
  const bool pk = K.packed;  // float2 accumulators of m3 pairs (fpath2)
  for (size_t k = 0; k < shapes.size(); ++k) {
    const int N1 = std::get<0>(shapes[k]), N3 = std::get<1>(shapes[k]);
    const int NA = pk ? (N3 + 1) / 2 : N3;  // accumulators
    const std::string FT = pk ? "float2" : "float";
    const bool full = std::get<2>(shapes[k]);
    o << "// shape " << k << ": one path " << N1 << " x " << N3 << ", one channel per lane" << (pk ? ", packed" : "")
      << "\n"
      << "__device__ __noinline__ void fgen_" << k
      << "(const int* __restrict__ rowptr, int n_recv, float* __restrict__ out, int* __restrict__ err,\n"
         "    unsigned char* smem, int u0, int chs, int choff, int wst, int xst, int ooff, int mul, int* qp) {\n"
         "  const int lane = threadIdx.x & 31;\n"
         "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
         "  const int u = u0 + lane;\n"
         "  const bool ok = " << (full ? "true" : "u < mul") << ";\n"
         "  (void)mul;\n"
         "  int q = *qp;\n"
         "#pragma unroll 1\n  for (int i = RECV_FIRST; i < RECV_END; i += RECV_STEP) {\n"
         "  const int e0 = EDGE_LO(i), e1 = EDGE_HI(i);\n"
         "  " << FT << " acc[" << NA << "];\n"
         "#pragma unroll\n  for (int k = 0; k < " << NA << "; ++k) acc[k] = " << (pk ? "make_float2(0.f, 0.f)" : "0.f")
      << ";\n"
         "#pragma unroll 1\n  for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
         "    const int s = q % NSTAGE;\n"
         "    if (!stage_ready(full0, s, (q / NSTAGE) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
         "    const int nb = min(NB, e1 - eb);\n"
         "    const unsigned char* st = stage_ptr(smem, s);\n"
         "    const float* sW = reinterpret_cast<const float*>(st + OFF_W) + wst;\n"
         "    const float* sX = reinterpret_cast<const float*>(st + OFF_X) + xst;\n"
         "    const float* sC = reinterpret_cast<const float*>(st + OFF_CH) + choff;\n"
         "#pragma unroll 1\n    for (int b = 0; b < nb; ++b) {\n"
         "      " << FT << " xv[1][" << N1 << "];\n      float w[1];\n"
         "#pragma unroll\n      for (int m1 = 0; m1 < " << N1 << "; ++m1) "
      << (pk ? "{ const float v = ok ? sX[b * XS + u * " + std::to_string(N1) + " + m1] : 0.f; xv[0][m1] = make_float2(v, v); }"
             : "xv[0][m1] = ok ? sX[b * XS + u * " + std::to_string(N1) + " + m1] : 0.f;")
      << "\n      w[0] = ok ? sW[b * WS + u] : 0.f;\n";
    const std::string fp = pk ? "2<" : "<";
    if (K.tangent)
      o << "      " << FT << " xtv[1][" << N1 << "];\n      float wt[1];\n"
           "      const float* sXt = reinterpret_cast<const float*>(st + OFF_XT) + xst;\n"
           "      const float* sWt = reinterpret_cast<const float*>(st + OFF_WT) + wst;\n"
           "      const float* sCt = reinterpret_cast<const float*>(st + OFF_CHT) + choff;\n"
           "#pragma unroll\n      for (int m1 = 0; m1 < " << N1 << "; ++m1) "
        << (pk ? "{ const float v = ok ? sXt[b * XS + u * " + std::to_string(N1) + " + m1] : 0.f; xtv[0][m1] = make_float2(v, v); }"
               : "xtv[0][m1] = ok ? sXt[b * XS + u * " + std::to_string(N1) + " + m1] : 0.f;")
        << "\n      wt[0] = ok ? sWt[b * WS + u] : 0.f;\n"
           "      fpath_tan" << fp << N1 << "," << N3 << ",1,0," << NA << ">(acc, sC + b * chs, sCt + b * chs, xv, xtv, w, wt);\n";
    else
      o << "      fpath" << fp << N1 << "," << N3 << ",1,0," << NA << ">(acc, sC + b * chs, xv, w);\n";
    o << "    }\n    __syncwarp();\n    if (lane == 0) mbar_arrive(empty0 + 8 * s);\n  }\n"
         "  if (ok) {\n    float* orow = out + (size_t)i * DOUT + ooff;\n"
         "#pragma unroll\n    for (int m3 = 0; m3 < " << N3 << "; ++m3) "
      << (K.accumulate ? "red_add(&orow[u * " : "orow[u * ") << N3 << " + m3]" << (K.accumulate ? ", " : " = ")
      << (pk ? "(m3 & 1) ? acc[m3 >> 1].y : acc[m3 >> 1].x" : "acc[m3]") << (K.accumulate ? ")" : "") << ";\n  }\n"
         "  }\n  *qp = q;\n}\n";
  }
  gen_fwd_idle(o);
  auto table = [&](const char* name, auto f) {
    o << "__constant__ int " << name << "[" << S * NW << "] = {";
    for (int s = 0; s < S; ++s)
      for (int w = 0; w < NW; ++w) o << (w < (int)F.slice_roles[s].size() ? f(s, F.slice_roles[s][w]) : 0) << ",";
    o << "};\n";
  };
  o << "__constant__ int kShape[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? shape_of[F.slice_roles[s][w]] : -1) << ",";
  o << "};\n";
  table("kU0", [&](int, int ri) { return P.fwd_roles[ri].u0; });
  table("kChOff", [&](int s, int ri) { return SL[s].ch_off.at(P.fwd_roles[ri].paths[0]); });
  table("kWst", [&](int s, int ri) { return SL[s].w_st.at(P.fwd_roles[ri].paths[0]); });
  table("kXst", [&](int s, int ri) { return SL[s].x_st.at(P.fwd_roles[ri].irrep); });
  table("kOoff", [&](int, int ri) { return P.paths[P.fwd_roles[ri].paths[0]].o_off; });
  table("kMul", [&](int, int ri) { return P.in[P.fwd_roles[ri].irrep].mul; });
  o << "__constant__ int kEntBegin[" << S + 1 << "] = {";
  for (int v : P.fwd_ent_begin) o << v << ",";
  o << "};\n";
  (void)slice_of;
  std::ostringstream d;
  for (size_t k = 0; k < shapes.size(); ++k)
    d << "    case " << k << ": fgen_" << k
      << "(rowptr, n_recv, out, err, smem, u0, chs, kChOff[slot], kWst[slot], kXst[slot], kOoff[slot], kMul[slot], "
         "&q); break;\n";
  gen_fwd_entry(o, kname, min_blocks, d.str(), K.tangent);
  return o.str();
}

static std::string gen_fwd_source(const Plan& P, const std::vector<SliceLayout>& SL, const KernelShape& K,
                                  const std::string& kname, int min_blocks) {
  const FwdConfig& F = P.fcfg;
  const int S = K.S, NW = K.nw;
  std::ostringstream o;
  o << spin_limit_define() << kPrelude;
  o << gen_common_device(P, SL, K, false);

  std::vector<int> slice_of(P.fwd_roles.size(), -1);
  for (int s = 0; s < S; ++s)
    for (int v : F.slice_roles[s]) slice_of[v] = s;
  if (F.generic) return gen_fwd_generic(P, SL, K, kname, min_blocks, o, slice_of);
  std::vector<int> shape_of(P.fwd_roles.size(), -1), shape_rep;
  for (size_t ri = 0; ri < P.fwd_roles.size(); ++ri) {
    const FwdRole& r = P.fwd_roles[ri];
    for (size_t k = 0; k < shape_rep.size(); ++k) {
      const FwdRole& q = P.fwd_roles[shape_rep[k]];
      if (q.irrep == r.irrep && q.R == r.R && q.paths == r.paths && slice_of[shape_rep[k]] == slice_of[ri]) {
        shape_of[ri] = (int)k;
        break;
      }
    }
    if (shape_of[ri] < 0) {
      shape_of[ri] = (int)shape_rep.size();
      shape_rep.push_back((int)ri);
    }
  }
  for (size_t k = 0; k < shape_rep.size(); ++k) {
    const FwdRole& r = P.fwd_roles[shape_rep[k]];
    const SliceLayout& sl = SL[slice_of[shape_rep[k]]];
    const Irrep& h = P.in[r.irrep];
    const int N1 = 2 * h.l + 1, R = r.R, MUL = h.mul;
    // accumulators: floats, or float2 pairs of consecutive m3 (packed)
    const bool pk = K.packed;
    auto np = [&](int pi) { return pk ? P.paths[pi].l3 + 1 : 2 * P.paths[pi].l3 + 1; };
    int nacc = 0;
    for (int pi : r.paths) nacc += R * np(pi);
    const std::string AT = pk ? "float2" : "float";
    o << "// shape " << k << ": irrep " << r.irrep << " (" << h.mul << "x" << h.l << "), " << r.paths.size()
      << " paths, R=" << R << (pk ? ", packed" : "") << "\n";
    o << "__device__ __noinline__ void fcons_" << k
      << "(const int* __restrict__ rowptr, int n_recv, float* __restrict__ out, int* __restrict__ err,\n"
         "    unsigned char* smem, int u0, int chs, int* qp) {\n"
         "  const int lane = threadIdx.x & 31;\n"
         "  const u32 full0 = smem_u32(smem), empty0 = full0 + NSTAGE * 8;\n"
         "  bool ok[" << R << "];\n"
         "#pragma unroll\n  for (int r = 0; r < " << R << "; ++r) ok[r] = "
      << (MUL % (32 * R) == 0 ? std::string("true") : "u0 + r * 32 + lane < " + std::to_string(MUL))
      << ";  // every lane holds a channel when the blocks are full\n"
         "  int q = *qp;\n"
         "#pragma unroll 1\n  for (int i = RECV_FIRST; i < RECV_END; i += RECV_STEP) {\n"
         "  const int e0 = EDGE_LO(i), e1 = EDGE_HI(i);\n"
         "  " << AT << " acc[" << nacc << "];\n"
         "#pragma unroll\n  for (int k = 0; k < " << nacc << "; ++k) acc[k] = "
      << (pk ? "make_float2(0.f, 0.f)" : "0.f") << ";\n"
         "#pragma unroll 1\n  for (int eb = e0; eb < e1; eb += NB, ++q) {\n"
         "    const int s = q % NSTAGE;\n"
         "    if (!stage_ready(full0, s, (q / NSTAGE) & 1)) { if (lane == 0) atomicOr(err, 10); *qp = -1; return; }\n"
         "    const int nb = min(NB, e1 - eb);\n"
         "    const unsigned char* st = stage_ptr(smem, s);\n"
         "    const float* sW = reinterpret_cast<const float*>(st + OFF_W);\n"
         "    const float* sX = reinterpret_cast<const float*>(st + OFF_X) + " << sl.x_st.at(r.irrep) << ";\n"
         "    const float* sC = reinterpret_cast<const float*>(st + OFF_CH);\n"
         "#pragma unroll 1\n    for (int b = 0; b < nb; ++b) {\n"
         "      const float* chb = sC + b * chs;\n"
         "      const float* wr = sW + b * WS;\n"
         "      const float* xr = sX + b * XS;\n"
         "      " << (pk ? "float2" : "float") << " xv[" << R << "][" << N1 << "];\n"
         "#pragma unroll\n      for (int r = 0; r < " << R << "; ++r) {\n"
         "        const int u = u0 + r * 32 + lane;\n"
         "#pragma unroll\n        for (int m1 = 0; m1 < " << N1 << "; ++m1) "
      << (pk ? "{ const float v = ok[r] ? xr[u * " + std::to_string(N1) + " + m1] : 0.f; xv[r][m1] = make_float2(v, v); }"
             : "xv[r][m1] = ok[r] ? xr[u * " + std::to_string(N1) + " + m1] : 0.f;")
      << "\n      }\n";
    if (K.tangent)  // the tangent copies of the same pieces
      o << "      const float* chtb = reinterpret_cast<const float*>(st + OFF_CHT) + b * chs;\n"
           "      const float* wtr = reinterpret_cast<const float*>(st + OFF_WT) + b * WS;\n"
           "      const float* xtr = reinterpret_cast<const float*>(st + OFF_XT) + " << sl.x_st.at(r.irrep)
        << " + b * XS;\n"
           "      " << (pk ? "float2" : "float") << " xtv[" << R << "][" << N1 << "];\n"
           "#pragma unroll\n      for (int r = 0; r < " << R << "; ++r) {\n"
           "        const int u = u0 + r * 32 + lane;\n"
           "#pragma unroll\n        for (int m1 = 0; m1 < " << N1 << "; ++m1) "
        << (pk ? "{ const float v = ok[r] ? xtr[u * " + std::to_string(N1) + " + m1] : 0.f; xtv[r][m1] = make_float2(v, v); }"
               : "xtv[r][m1] = ok[r] ? xtr[u * " + std::to_string(N1) + " + m1] : 0.f;")
        << "\n      }\n";
    int A = 0;
    for (int pi : r.paths) {
      const Path& p = P.paths[pi];
      const int N3 = 2 * p.l3 + 1;
      o << "      { float w[" << R << "];\n#pragma unroll\n        for (int r = 0; r < " << R
        << "; ++r) w[r] = ok[r] ? wr[" << sl.w_st.at(pi) << " + u0 + r * 32 + lane] : 0.f;\n";
      if (K.tangent)
        o << "        float wt[" << R << "];\n#pragma unroll\n        for (int r = 0; r < " << R
          << "; ++r) wt[r] = ok[r] ? wtr[" << sl.w_st.at(pi) << " + u0 + r * 32 + lane] : 0.f;\n"
          << "        fpath_tan" << (pk ? "2<" : "<") << N1 << "," << N3 << "," << R << "," << A << "," << nacc
          << ">(acc, chb + " << sl.ch_off.at(pi) << ", chtb + " << sl.ch_off.at(pi) << ", xv, xtv, w, wt); }\n";
      else
        o << "        fpath" << (pk ? "2<" : "<") << N1 << "," << N3 << "," << R << "," << A << "," << nacc
          << ">(acc, chb + " << sl.ch_off.at(pi) << ", xv, w); }\n";
      A += R * np(pi);
    }
    o << "    }\n    __syncwarp();\n    if (lane == 0) mbar_arrive(empty0 + 8 * s);\n  }\n";
    o << "  float* orow = out + (size_t)i * DOUT;\n";
    A = 0;
    for (int pi : r.paths) {
      const Path& p = P.paths[pi];
      const int N3 = 2 * p.l3 + 1;
      o << "#pragma unroll\n  for (int r = 0; r < " << R << "; ++r) if (ok[r]) {\n    const int u = u0 + r * 32 + lane;\n"
        << "#pragma unroll\n    for (int m3 = 0; m3 < " << N3 << "; ++m3) " << (K.accumulate ? "red_add(&orow[" : "orow[")
        << p.o_off << " + u * " << N3
        << " + m3]" << (K.accumulate ? ", " : " = ")
        << (pk ? "(m3 & 1) ? acc[" + std::to_string(A) + " + r * " + std::to_string(np(pi)) + " + (m3 >> 1)].y : acc[" +
                     std::to_string(A) + " + r * " + std::to_string(np(pi)) + " + (m3 >> 1)].x"
               : "acc[" + std::to_string(A) + " + r * " + std::to_string(N3) + " + m3]")
        << (K.accumulate ? ")" : "") << ";\n  }\n";
      A += R * np(pi);
    }
    o << "  }\n  *qp = q;\n}\n";
  }
  gen_fwd_idle(o);
  o << "__constant__ int kShape[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? shape_of[F.slice_roles[s][w]] : -1) << ",";
  o << "};\n__constant__ int kU0[" << S * NW << "] = {";
  for (int s = 0; s < S; ++s)
    for (int w = 0; w < NW; ++w)
      o << (w < (int)F.slice_roles[s].size() ? P.fwd_roles[F.slice_roles[s][w]].u0 : 0) << ",";
  o << "};\n__constant__ int kEntBegin[" << S + 1 << "] = {";
  for (int v : P.fwd_ent_begin) o << v << ",";
  o << "};\n";
  std::ostringstream d;
  for (size_t k = 0; k < shape_rep.size(); ++k)
    d << "    case " << k << ": fcons_" << k << "(rowptr, n_recv, out, err, smem, u0, chs, &q); break;\n";
  gen_fwd_entry(o, kname, min_blocks, d.str(), K.tangent);
  return o.str();
}

// Instructions one warp issues per edge for a role (FMAs, shared loads).
static double fwd_role_cost(const Plan& P, const FwdRole& r) {
  const int n1 = 2 * P.in[r.irrep].l + 1;
  double c = (double)r.R * n1;  // x
  for (int pi : r.paths) {
    const int n3 = 2 * P.paths[pi].l3 + 1;
    const double fma = n1 == 1 ? 1 + n3 : (n1 < n3 ? n1 + n1 * n3 : n1 * n3 + n3);
    c += r.R * (fma + 1) + (double)n3 * ((n1 + 3) / 4);
  }
  return c;
}

// The staging layout of each forward slice: the paths and hidden irreps of
// its roles.
static std::vector<SliceLayout> forward_slices(const Plan& P, bool m1_major) {
  const FwdConfig& F = P.fcfg;
  std::vector<SliceLayout> SL(F.S);
  for (int s = 0; s < F.S; ++s) {
    SL[s].m1_major = m1_major;
    std::vector<char> pseen(P.paths.size(), 0), iseen(P.in.size(), 0);
    for (int ri : F.slice_roles[s]) {
      for (int pi : P.fwd_roles[ri].paths) pseen[pi] = 1;
      iseen[P.fwd_roles[ri].irrep] = 1;
    }
    for (size_t k = 0; k < P.paths.size(); ++k)
      if (pseen[k]) SL[s].paths.push_back((int)k);
    for (size_t a = 0; a < P.in.size(); ++a)
      if (iseen[a]) SL[s].irreps.push_back((int)a);
    layout_slice(P, SL[s], false);
  }
  return SL;
}

cgtp_status build_forward(Plan& P) {
  // ---- roles: per hidden irrep, channel blocks x path groups
  // accumulator budget per lane (tuning override CGTP_FWD_BUDGET)
  int kAccBudget = 64;
  if (const char* v = std::getenv("CGTP_FWD_BUDGET")) kAccBudget = std::max(13, std::min(128, std::atoi(v)));
  int force_R = 0;  // channels per lane (tuning override CGTP_FWD_R: 1 or 2)
  if (const char* v = std::getenv("CGTP_FWD_R")) force_R = std::max(1, std::min(2, std::atoi(v)));
  P.fwd_roles.clear();
  for (size_t a = 0; a < P.in.size(); ++a) {
    const Irrep& h = P.in[a];
    std::vector<int> ps;
    for (size_t k = 0; k < P.paths.size(); ++k)
      if (P.paths[k].irrep == (int)a) ps.push_back((int)k);
    if (ps.empty()) continue;
    // wide inputs (l >= 3): one channel per lane and fewer accumulators, so
    // that x, w*x and the Chat row still fit beside them without spilling
    const int n1 = 2 * h.l + 1;
    const int R = force_R ? std::min(force_R, std::max(1, h.mul / 32)) : ((h.mul >= 64 && h.l < 3) ? 2 : 1);
    const int beta = h.l < 3 ? std::max(13, kAccBudget / R)
                             : std::max(13, kAccBudget - 2 * n1 - ((n1 + 3) & ~3));
    std::vector<std::vector<int>> groups;
    int sum = 0;
    for (int pi : ps) {
      const int n3 = 2 * P.paths[pi].l3 + 1;
      if (groups.empty() || sum + n3 > beta) {
        groups.push_back({});
        sum = 0;
      }
      groups.back().push_back(pi);
      sum += n3;
    }
    const int nblk = (h.mul + 32 * R - 1) / (32 * R);
    (void)n1;
    for (auto& g : groups)
      for (int blk = 0; blk < nblk; ++blk) {
        FwdRole r;
        r.irrep = (int)a;
        r.u0 = blk * 32 * R;
        r.R = R;
        r.paths = g;
        r.cost = fwd_role_cost(P, r);
        P.fwd_roles.push_back(r);
      }
  }
  // Balanced roles (CGTP_FWD_BALANCE=1): per hidden irrep, the channels per
  // lane and the runs of its paths chosen so that the costliest role is as
  // cheap as the warp budget allows (one slice of at most 16 warps, 8 with
  // inputs of l >= 3).  A stage is released only when every warp has
  // finished it, so the costliest role sets the pace.
  if (const char* v = std::getenv("CGTP_FWD_BALANCE"); v && *v == '1') {
    bool wide_in = false;
    for (auto& h : P.in) wide_in = wide_in || h.l >= 3;
    const int cap_roles = wide_in ? 8 : 16;
    struct Opt {
      int a, R, nblk;
      std::vector<int> ps;
      int acc_cap;
    };
    std::vector<Opt> opts;
    for (size_t a = 0; a < P.in.size(); ++a) {
      const Irrep& h = P.in[a];
      std::vector<int> ps;
      for (size_t k = 0; k < P.paths.size(); ++k)
        if (P.paths[k].irrep == (int)a) ps.push_back((int)k);
      if (ps.empty()) continue;
      const int n1 = 2 * h.l + 1;
      for (int R = 1; R <= 2; ++R) {
        if (R == 2 && (h.mul < 64 || h.l >= 3)) continue;
        const int cap = h.l < 3 ? kAccBudget : std::max(13, kAccBudget - 2 * n1 - ((n1 + 3) & ~3));
        opts.push_back({(int)a, R, (h.mul + 32 * R - 1) / (32 * R), ps, cap});
      }
    }
    auto run_cost = [&](const Opt& o, size_t i, size_t j) {
      FwdRole r;
      r.irrep = o.a;
      r.u0 = 0;
      r.R = o.R;
      r.paths.assign(o.ps.begin() + i, o.ps.begin() + j);
      return fwd_role_cost(P, r);
    };
    // the greedy runs of an option under a cost bound T (empty: infeasible)
    auto groups_for = [&](const Opt& o, double T) {
      std::vector<std::pair<size_t, size_t>> g;
      size_t i = 0;
      while (i < o.ps.size()) {
        size_t j = i;
        int acc = 0;
        while (j < o.ps.size()) {
          const int add = o.R * (2 * P.paths[o.ps[j]].l3 + 1);
          if (j > i && (acc + add > o.acc_cap || run_cost(o, i, j + 1) > T)) break;
          acc += add;
          ++j;
        }
        if (run_cost(o, i, j) > T) return std::vector<std::pair<size_t, size_t>>();
        g.push_back({i, j});
        i = j;
      }
      return g;
    };
    std::vector<double> cand;
    for (auto& o : opts)
      for (size_t i = 0; i < o.ps.size(); ++i)
        for (size_t j = i + 1; j <= o.ps.size(); ++j) cand.push_back(run_cost(o, i, j));
    std::sort(cand.begin(), cand.end());
    cand.erase(std::unique(cand.begin(), cand.end()), cand.end());
    std::vector<FwdRole> best;
    for (double T : cand) {
      std::vector<FwdRole> roles;
      bool ok = true;
      for (size_t a = 0; a < P.in.size() && ok; ++a) {
        int best_n = -1;
        const Opt* bo = nullptr;
        std::vector<std::pair<size_t, size_t>> bg;
        for (auto& o : opts) {
          if (o.a != (int)a) continue;
          auto g = groups_for(o, T);
          if (g.empty()) continue;
          const int n = (int)g.size() * o.nblk;
          if (best_n < 0 || n < best_n || (n == best_n && o.R > bo->R)) {
            best_n = n;
            bo = &o;
            bg = g;
          }
        }
        bool has_paths = false;
        for (auto& o : opts) has_paths = has_paths || o.a == (int)a;
        if (!has_paths) continue;
        if (!bo) {
          ok = false;
          break;
        }
        for (auto& gr : bg)
          for (int blk = 0; blk < bo->nblk; ++blk) {
            FwdRole r;
            r.irrep = bo->a;
            r.u0 = blk * 32 * bo->R;
            r.R = bo->R;
            r.paths.assign(bo->ps.begin() + gr.first, bo->ps.begin() + gr.second);
            r.cost = fwd_role_cost(P, r);
            roles.push_back(r);
          }
      }
      if (ok && (int)roles.size() <= cap_roles) {
        best = roles;
        break;
      }
    }
    if (!best.empty()) P.fwd_roles = best;
  }
  // Roles are not split further to balance them: measured on B200, more and
  // smaller roles (single-block channel groups, split path groups) made the
  // forward slower (more distinct code resident at once, x and Chat read by
  // more warps), so the coarse roles above stand.
  const int NR = (int)P.fwd_roles.size();
  FwdConfig& F = P.fcfg;
  F = FwdConfig();
  if (NR == 0) return CGTP_OK;  // no paths: forward writes zeros
  // Wide plans (an input of l >= 3 and more than 16 coarse roles): the coarse
  // roles' fully unrolled multi-path code outgrows the instruction cache
  // (measured on B200: most cycles stalled on instruction fetch).  There a
  // role is one path and one block of 32 channels, and roles of the same
  // (2l1+1, 2l3+1) shape share one function with the path's offsets as
  // arguments; slices take roles in (shape, irrep) order, 8 per slice.
  bool wide = false;
  for (auto& r : P.fwd_roles) wide = wide || P.in[r.irrep].l >= 3;
  F.generic = wide && NR > 16;
  std::vector<FwdRole> roles;
  if (F.generic) {
    for (size_t k = 0; k < P.paths.size(); ++k) {
      const Path& p = P.paths[k];
      const int mul = P.in[p.irrep].mul;
      for (int u0 = 0; u0 < mul; u0 += 32) {
        FwdRole r;
        r.irrep = p.irrep;
        r.u0 = u0;
        r.R = 1;
        r.paths = {(int)k};
        r.cost = fwd_role_cost(P, r);
        roles.push_back(r);
      }
    }
    auto key = [&](const FwdRole& r) {
      const Path& p = P.paths[r.paths[0]];
      return std::make_tuple(-(2 * P.in[r.irrep].l + 1) * (2 * p.l3 + 1), 2 * P.in[r.irrep].l + 1, 2 * p.l3 + 1,
                             r.irrep, r.paths[0], r.u0);
    };
    std::stable_sort(roles.begin(), roles.end(), [&](const FwdRole& a, const FwdRole& b) { return key(a) < key(b); });
    P.fwd_roles = roles;
  }
  const int NR2 = (int)P.fwd_roles.size();
  if (F.generic) {
    int per = 8;  // roles (consumer warps) per slice
    if (const char* v = std::getenv("CGTP_FWD_GENERIC_WARPS")) per = std::max(1, std::min(16, std::atoi(v)));
    F.S = (NR2 + per - 1) / per;
    F.slice_roles.assign(F.S, {});
    for (int ri = 0; ri < NR2; ++ri) F.slice_roles[ri / per].push_back(ri);
  } else {
    // up to 16 consumer warps per CTA; 8 when the roles are register-heavy
    // (wide inputs), so that two CTAs of (8 + 2) warps keep 96 registers each
    int kMaxWarps = 16;
    for (auto& r : P.fwd_roles)
      if (P.in[r.irrep].l >= 3 && NR > 8) kMaxWarps = 8;
    F.S = (NR + kMaxWarps - 1) / kMaxWarps;
    // longest-processing-time assignment of roles to slices
    std::vector<int> order(NR);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return P.fwd_roles[a].cost > P.fwd_roles[b].cost; });
    const int cap = (NR + F.S - 1) / F.S;
    F.slice_roles.assign(F.S, {});
    std::vector<double> load(F.S, 0.0);
    for (int ri : order) {
      int best = -1;
      for (int s = 0; s < F.S; ++s)
        if ((int)F.slice_roles[s].size() < cap && (best < 0 || load[s] < load[best])) best = s;
      F.slice_roles[best].push_back(ri);
      load[best] += P.fwd_roles[ri].cost;
    }
    for (auto& v : F.slice_roles) std::sort(v.begin(), v.end());
  }
  F.nw = 0;
  for (auto& v : F.slice_roles) F.nw = std::max<int>(F.nw, (int)v.size());
  F.nacc = 1;
  for (auto& r : P.fwd_roles) {
    int n = 0;
    for (int pi : r.paths) n += r.R * (2 * P.paths[pi].l3 + 1);
    F.nacc = std::max(F.nacc, n);
  }
  // Packed roles (float2 accumulators of m3 pairs, m1-major Chat) for plans
  // with a hidden irrep of l >= 3, whose long m3 rows pack well.  Measured on
  // B200: Lmax 3 470 -> 433 us, Case 5 470 -> 402 us, Lmax 6 2035 -> 1631 us,
  // Case 6 821 -> 721 us, Case 4 unchanged; plans with l <= 2 inputs lose
  // (Lmax 2 35 -> 43 us, Lmax 2 wide 137 -> 148 us).
  int lmax_in = 0;
  for (const Irrep& h : P.in) lmax_in = std::max(lmax_in, h.l);
  F.packed = P.fwd_packed < 0 ? lmax_in >= 3 : P.fwd_packed == 1;
  std::vector<SliceLayout> SL = forward_slices(P, F.packed);
  KernelShape K;
  K.S = F.S;
  K.nw = F.nw;
  K.WB = 0;  // output rows go straight from registers to global memory
  K.packed = F.packed;
  // tuning overrides for the plain forward alone: edges per chunk and ring depth
  if (const char* v = std::getenv("CGTP_FWD_CHUNK")) K.force_B = std::max(1, std::min(8, std::atoi(v)));
  if (const char* v = std::getenv("CGTP_FWD_STAGES")) K.force_stages = std::max(2, std::min(6, std::atoi(v)));
  plan_layout(P, SL, K, false);
  F.B = K.B;
  F.stages = K.stages;
  F.w_smem = K.w_bulk;
  F.x_smem = K.x_bulk;

  cgtp_status st = upload_chat_tables(P, SL, &P.d_fwd_ent, P.fwd_ent_begin);
  if (st != CGTP_OK) return st;
  for (size_t k = 0; k + 1 < P.fwd_ent_begin.size(); ++k)
    K.rec_max = std::max(K.rec_max, P.fwd_ent_begin[k + 1] - P.fwd_ent_begin[k]);
  const std::string name = "cgtp_fwd";
  // register cap from the resident CTAs shared memory allows; one CTA fewer
  // (but not below two) when the compiler reports sizeable spills
  if (K.smem > 227 * 1024) return fail(CGTP_ERR_SIZE, "forward kernel needs too much shared memory");
  bool fixed = false;
  int mb0 = initial_min_blocks(K.smem, &fixed);
  if (const char* v = std::getenv("CGTP_FWD_MIN_BLOCKS")) {
    mb0 = std::max(1, std::atoi(v));
    fixed = true;
  }
  const int mb_floor = fixed ? mb0 : std::min(mb0, 2);
  // The compile runs on a host thread while the backward is planned and
  // compiled (NVRTC needs no CUDA context); finish_forward joins and loads.
  // It reads only the plan's paths, irreps and forward fields, all set by now.
  auto pend = std::make_unique<PendingCompile>();
  PendingCompile* pc = pend.get();
  const Plan& CP = P;
  auto body = [pc, &CP, SL, K, mb0, mb_floor, name]() {
    try {
      for (int mb = mb0; mb >= mb_floor; --mb) {
        pc->src = gen_fwd_source(CP, SL, K, name, mb);
        pc->st = jit_build(pc->src, name, pc->bin);
        if (pc->st != CGTP_OK || mb == mb_floor || max_spill_bytes(pc->bin.log) <= 64) break;
      }
    } catch (const std::exception& e) {
      pc->st = CGTP_ERR_OOM;
      pc->bin.err = std::string("exception while building the forward: ") + e.what();
    }
  };
  try {
    pend->th = std::thread(body);
  } catch (...) {
    body();
  }
  P.fwd.threads = (F.nw + 2) * 32;
  P.fwd.smem = K.smem;
  P.fwd_pending = std::move(pend);
  return CGTP_OK;
}

// The forward's tangent kernel (cgtp_fwd_tan): the same roles and slices,
// every W, x and Y piece staged with its directional derivative, so that one
// pass gives d/dt fwd(x + t xt, Y + t Yt, W + t Wt).  Built on first use.
cgtp_status build_forward_tangent(Plan& P, JitKernel& out, std::string* src_out) {
  const FwdConfig& F = P.fcfg;
  std::vector<SliceLayout> SL = forward_slices(P, F.packed);  // the plain forward's Chat records
  KernelShape K;
  K.S = F.S;
  K.nw = F.nw;
  K.WB = 0;
  K.tangent = true;
  K.packed = F.packed;
  // tuning overrides for this kernel alone: edges per chunk and ring depth
  if (const char* v = std::getenv("CGTP_FWD_TAN_CHUNK")) K.force_B = std::max(1, std::min(8, std::atoi(v)));
  if (const char* v = std::getenv("CGTP_FWD_TAN_STAGES")) K.force_stages = std::max(2, std::min(6, std::atoi(v)));
  plan_layout(P, SL, K, false);
  for (size_t k = 0; k + 1 < P.fwd_ent_begin.size(); ++k)
    K.rec_max = std::max(K.rec_max, P.fwd_ent_begin[k + 1] - P.fwd_ent_begin[k]);
  if (K.smem > 227 * 1024) return fail(CGTP_ERR_SIZE, "tangent forward needs too much shared memory");
  bool fixed = false;
  const int mb0 = initial_min_blocks(K.smem, &fixed);
  const int mb_floor = fixed ? mb0 : std::min(mb0, 2);
  const std::string name = "cgtp_fwd_tan";
  std::string src;
  JitBinary bin;
  cgtp_status st = CGTP_OK;
  for (int mb = mb0; mb >= mb_floor; --mb) {
    src = gen_fwd_source(P, SL, K, name, mb);
    st = jit_build(src, name, bin);
    if (st != CGTP_OK || mb == mb_floor || max_spill_bytes(bin.log) <= 64) break;
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

// The accumulating forward (cgtp_fwd_acc): the plain forward's roles, slices
// and layout, adding its result to the output rows.  The double backward sums
// three forwards with it where that beats the tangent forward.  Built on
// first use.
cgtp_status build_forward_accumulate(Plan& P, JitKernel& out, std::string* src_out) {
  const FwdConfig& F = P.fcfg;
  std::vector<SliceLayout> SL = forward_slices(P, F.packed);
  KernelShape K;
  K.S = F.S;
  K.nw = F.nw;
  K.WB = 0;
  K.packed = F.packed;
  K.accumulate = true;
  plan_layout(P, SL, K, false);
  for (size_t k = 0; k + 1 < P.fwd_ent_begin.size(); ++k)
    K.rec_max = std::max(K.rec_max, P.fwd_ent_begin[k + 1] - P.fwd_ent_begin[k]);
  if (K.smem > 227 * 1024) return fail(CGTP_ERR_SIZE, "forward kernel needs too much shared memory");
  bool fixed = false;
  const int mb0 = initial_min_blocks(K.smem, &fixed);
  const int mb_floor = fixed ? mb0 : std::min(mb0, 2);
  const std::string name = "cgtp_fwd_acc";
  std::string src;
  JitBinary bin;
  cgtp_status st = CGTP_OK;
  for (int mb = mb0; mb >= mb_floor; --mb) {
    src = gen_fwd_source(P, SL, K, name, mb);
    st = jit_build(src, name, bin);
    if (st != CGTP_OK || mb == mb_floor || max_spill_bytes(bin.log) <= 64) break;
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

cgtp_status finish_forward(Plan& P) {
  if (!P.fwd_pending) return CGTP_OK;
  std::unique_ptr<PendingCompile> pc = std::move(P.fwd_pending);
  pc->join();
  if (pc->st != CGTP_OK) {
    set_error(pc->bin.err);
    return pc->st;
  }
  const cgtp_status st = jit_load(pc->bin, "cgtp_fwd", P.fwd);
  if (st != CGTP_OK) return st;
  if (const char* d = std::getenv("CGTP_DUMP_SOURCE")) {
    FILE* f = std::fopen((std::string(d) + "/fwd.cu").c_str(), "w");
    if (f) {
      std::fputs(pc->src.c_str(), f);
      std::fclose(f);
    }
  }
  return CGTP_OK;
}

}  // namespace cgtp
