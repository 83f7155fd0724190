// plan.cpp -- path enumeration, layout offsets and the division of the
// work into warp roles.
//
// Path rule (the reading of LunaTP, arXiv 2610.18393, Table 1 that
// reproduces all six of its output multiplicities): for each hidden irrep
// (u, l1, p1) in order, each edge irrep (l2, p2) in order, each l3 from
// |l1-l2| to l1+l2 ascending, the path exists when (l3, p1 p2) is an output
// irrep; its u channels are appended to that output block.
#include <algorithm>
#include <cmath>
#include <numeric>

#include "internal.hpp"

namespace cgtp {

cgtp_status build_paths(Plan& P) {
  std::string err;
  if (!parse_irreps(P.irreps_in_s.c_str(), P.in, err) ||
      !parse_irreps(P.irreps_edge_s.c_str(), P.edge, err) ||
      !parse_irreps(P.irreps_out_s.c_str(), P.out, err))
    return fail(CGTP_ERR_IRREPS_PARSE, err);
  if (P.lmax < 0 || P.lmax > 6) return fail(CGTP_ERR_LMAX, "lmax must be in 0..6");
  for (auto* v : {&P.in, &P.edge, &P.out})
    for (const auto& ir : *v)
      if (ir.l > P.lmax) return fail(CGTP_ERR_LMAX, "an irrep degree exceeds lmax");
  for (size_t k = 0; k < P.edge.size(); ++k)
    if (P.edge[k].mul != 1 || P.edge[k].l != (int)k)
      return fail(CGTP_ERR_IRREPS_PARSE, "edge irreps must be 1x0+1x1+...+1xL in order");
  for (size_t a = 0; a < P.out.size(); ++a)
    for (size_t b = a + 1; b < P.out.size(); ++b)
      if (P.out[a].l == P.out[b].l && P.out[a].parity == P.out[b].parity)
        return fail(CGTP_ERR_IRREPS_PARSE, "an (l, parity) appears twice in the output irreps");
  for (const auto& ir : P.in)
    if (ir.mul <= 0) return fail(CGTP_ERR_IRREPS_PARSE, "hidden multiplicities must be positive");

  P.L = (int)P.edge.size() - 1;
  P.D_e = (int64_t)(P.L + 1) * (P.L + 1);
  P.x_off.clear();
  int64_t off = 0;
  for (const auto& ir : P.in) {
    P.x_off.push_back((int)off);
    off += (int64_t)ir.mul * (2 * ir.l + 1);
  }
  P.D_in = off;
  P.out_off.clear();
  P.chan_base.clear();
  off = 0;
  int64_t cb = 0;
  for (const auto& ir : P.out) {
    P.out_off.push_back((int)off);
    P.chan_base.push_back((int)cb);
    off += (int64_t)ir.mul * (2 * ir.l + 1);
    cb += ir.mul;
  }
  P.D_out = off;
  P.U = cb;
  if (P.D_in >= (1 << 30) || P.D_out >= (1 << 30)) return fail(CGTP_ERR_SIZE, "irreps too wide");

  std::vector<int> filled(P.out.size(), 0);
  P.paths.clear();
  P.coeff.clear();
  for (size_t a = 0; a < P.in.size(); ++a) {
    const Irrep& h = P.in[a];
    for (const Irrep& ed : P.edge) {
      for (int l3 = std::abs(h.l - ed.l); l3 <= h.l + ed.l; ++l3) {
        const int par = h.parity * ed.parity;
        int o = -1;
        for (size_t q = 0; q < P.out.size(); ++q)
          if (P.out[q].l == l3 && P.out[q].parity == par) o = (int)q;
        if (o < 0) continue;
        Path p;
        p.l1 = h.l;
        p.l2 = ed.l;
        p.l3 = l3;
        p.irrep = (int)a;
        p.mul = h.mul;
        p.x_off = P.x_off[a];
        p.k0 = P.chan_base[o] + filled[o];
        p.o_off = P.out_off[o] + filled[o] * (2 * l3 + 1);
        p.out_irrep = o;
        p.c_off = (int)P.coeff.size();
        filled[o] += h.mul;
        std::vector<double> C;
        real_cg_block(h.l, ed.l, l3, C);
        P.coeff.insert(P.coeff.end(), C.begin(), C.end());
        P.paths.push_back(p);
      }
    }
  }
  for (size_t o = 0; o < P.out.size(); ++o)
    if (filled[o] != P.out[o].mul)
      return fail(CGTP_ERR_IRREPS_MISMATCH,
                  "output irrep " + std::to_string(P.out[o].mul) + "x" + std::to_string(P.out[o].l) +
                      (P.out[o].parity > 0 ? "e" : "o") + " receives " + std::to_string(filled[o]) +
                      " channels from the paths");
  return CGTP_OK;
}

}  // namespace cgtp
