// cg.cpp -- irreps parsing and the real Clebsch-Gordan blocks of the plan.
//
// The coefficients are built constructively with angular-momentum ladder
// operators (the "highest weight then lower" construction of the coupled
// states), not from a closed-form sum:
//   1. the top state |J J> = sum_m1 a(m1) |j1 m1>|j2 J-m1> is fixed by
//      J+|J J> = 0, which gives a two-term recurrence in m1 started at
//      m1 = j1 with a positive coefficient (Condon-Shortley), then normalised;
//   2. every lower state follows from J-|J M> = sqrt(J(J+1)-M(M-1)) |J M-1>
//      with J- = J1- + J2-.
// The complex coefficients are then moved to the real basis of the library's
// spherical harmonics (m>0: (Y_-m + (-1)^m Y_m)/sqrt2, m<0:
// i (Y_m - (-1)^m Y_-m)/sqrt2), the vanishing real or imaginary part is
// dropped, the block is scaled to sum C^2 = 2 l3 + 1 and its sign fixed so the
// first entry with |C| > 1e-12 (lexicographic m1, m2, m3) is positive.
#include <cctype>
#include <cmath>
#include <complex>
#include <cstring>

#include "internal.hpp"

namespace cgtp {

bool parse_irreps(const char* s, std::vector<Irrep>& out, std::string& err) {
  out.clear();
  if (!s) {
    err = "null irreps string";
    return false;
  }
  const char* p = s;
  while (true) {
    while (std::isspace((unsigned char)*p)) ++p;
    if (!std::isdigit((unsigned char)*p)) {
      err = std::string("expected a multiplicity in '") + s + "'";
      return false;
    }
    long mul = 0;
    while (std::isdigit((unsigned char)*p)) {
      mul = mul * 10 + (*p - '0');
      if (mul > (1 << 20)) {
        err = "multiplicity too large";
        return false;
      }
      ++p;
    }
    while (std::isspace((unsigned char)*p)) ++p;
    if (*p != 'x') {
      err = std::string("expected 'x' in '") + s + "'";
      return false;
    }
    ++p;
    while (std::isspace((unsigned char)*p)) ++p;
    if (!std::isdigit((unsigned char)*p)) {
      err = std::string("expected a degree in '") + s + "'";
      return false;
    }
    long l = 0;
    while (std::isdigit((unsigned char)*p)) {
      l = l * 10 + (*p - '0');
      if (l > 64) {
        err = "degree too large";
        return false;
      }
      ++p;
    }
    while (std::isspace((unsigned char)*p)) ++p;
    int par;
    if (*p == 'e')
      par = 1;
    else if (*p == 'o')
      par = -1;
    else {
      err = std::string("expected parity 'e' or 'o' in '") + s + "'";
      return false;
    }
    ++p;
    out.push_back({(int)mul, (int)l, par});
    while (std::isspace((unsigned char)*p)) ++p;
    if (*p == '\0') break;
    if (*p != '+') {
      err = std::string("unexpected character in '") + s + "'";
      return false;
    }
    ++p;
  }
  return true;
}

namespace {

// J+ |j m> = up(j,m) |j m+1>,  J- |j m> = dn(j,m) |j m-1>
inline double up(int j, int m) { return std::sqrt(double(j * (j + 1) - m * (m + 1))); }
inline double dn(int j, int m) { return std::sqrt(double(j * (j + 1) - m * (m - 1))); }

// complex CG <j1 m1 j2 m2 | J M> stored at [(m1+j1)*n2 + (m2+j2)]*n3 + (M+J)
void ladder_cg(int j1, int j2, int J, std::vector<double>& cg) {
  const int n1 = 2 * j1 + 1, n2 = 2 * j2 + 1, n3 = 2 * J + 1;
  cg.assign((size_t)n1 * n2 * n3, 0.0);
  auto at = [&](int m1, int m2, int M) -> double& {
    return cg[((size_t)(m1 + j1) * n2 + (m2 + j2)) * n3 + (M + J)];
  };
  // top state
  std::vector<double> a(n1, 0.0);
  const int lo = std::max(-j1, J - j2);
  a[j1 + j1] = 1.0;
  for (int m1 = j1 - 1; m1 >= lo; --m1)
    a[m1 + j1] = -a[m1 + 1 + j1] * up(j2, J - m1 - 1) / up(j1, m1);
  double nrm = 0.0;
  for (double v : a) nrm += v * v;
  nrm = std::sqrt(nrm);
  for (int m1 = lo; m1 <= j1; ++m1) at(m1, J - m1, J) = a[m1 + j1] / nrm;
  // lower
  for (int M = J; M > -J; --M) {
    const double inv = 1.0 / dn(J, M);
    for (int m1 = -j1; m1 <= j1; ++m1) {
      const int m2 = M - 1 - m1;
      if (m2 < -j2 || m2 > j2) continue;
      double v = 0.0;
      if (m1 + 1 <= j1) v += at(m1 + 1, m2, M) * dn(j1, m1 + 1);
      if (m2 + 1 <= j2) v += at(m1, m2 + 1, M) * dn(j2, m2 + 1);
      at(m1, m2, M - 1) = v * inv;
    }
  }
}

// row m (real index m+l) of the complex -> real change of basis
void real_basis(int l, std::vector<std::complex<double>>& U) {
  const int n = 2 * l + 1;
  const double h = 1.0 / std::sqrt(2.0);
  U.assign((size_t)n * n, {0.0, 0.0});
  for (int m = -l; m <= l; ++m) {
    const double sgn = (std::abs(m) % 2) ? -1.0 : 1.0;
    auto row = [&](int c) -> std::complex<double>& { return U[(size_t)(m + l) * n + (c + l)]; };
    if (m == 0) {
      row(0) = 1.0;
    } else if (m > 0) {
      row(-m) = h;
      row(m) = sgn * h;
    } else {
      row(m) = std::complex<double>(0.0, h);
      row(-m) = std::complex<double>(0.0, -sgn * h);
    }
  }
}

}  // namespace

bool real_cg_block(int l1, int l2, int l3, std::vector<double>& C) {
  if (l1 < 0 || l2 < 0 || l3 < std::abs(l1 - l2) || l3 > l1 + l2) return false;
  const int n1 = 2 * l1 + 1, n2 = 2 * l2 + 1, n3 = 2 * l3 + 1;
  std::vector<double> cg;
  ladder_cg(l1, l2, l3, cg);
  std::vector<std::complex<double>> U1, U2, U3;
  real_basis(l1, U1);
  real_basis(l2, U2);
  real_basis(l3, U3);
  const size_t nt = (size_t)n1 * n2 * n3;
  std::vector<std::complex<double>> Z(nt);
  // Z[a,b,c] = sum conj(U1[a,m1']) conj(U2[b,m2']) U3[c,m1'+m2'] cg[m1',m2',m1'+m2']
  for (int a = 0; a < n1; ++a)
    for (int b = 0; b < n2; ++b)
      for (int c = 0; c < n3; ++c) {
        std::complex<double> s = 0.0;
        for (int p1 = 0; p1 < n1; ++p1) {
          const auto u1 = std::conj(U1[(size_t)a * n1 + p1]);
          if (u1 == 0.0) continue;
          for (int p2 = 0; p2 < n2; ++p2) {
            const auto u2 = std::conj(U2[(size_t)b * n2 + p2]);
            if (u2 == 0.0) continue;
            const int M = (p1 - l1) + (p2 - l2);
            if (M < -l3 || M > l3) continue;
            const auto u3 = U3[(size_t)c * n3 + (M + l3)];
            if (u3 == 0.0) continue;
            s += u1 * u2 * u3 * cg[((size_t)p1 * n2 + p2) * n3 + (M + l3)];
          }
        }
        Z[((size_t)a * n2 + b) * n3 + c] = s;
      }
  double re2 = 0.0, im2 = 0.0;
  for (const auto& z : Z) {
    re2 += z.real() * z.real();
    im2 += z.imag() * z.imag();
  }
  const bool use_re = re2 >= im2;
  const double scale = std::sqrt(double(n3) / (use_re ? re2 : im2));
  C.resize(nt);
  for (size_t t = 0; t < nt; ++t) C[t] = (use_re ? Z[t].real() : Z[t].imag()) * scale;
  for (size_t t = 0; t < nt; ++t) {
    if (std::fabs(C[t]) > 1e-12) {
      if (C[t] < 0)
        for (auto& v : C) v = -v;
      break;
    }
  }
  // entries that vanish by symmetry come out of the ladder recursion as
  // rounding noise (~1e-14); every genuine entry for l <= 12 is far larger
  for (auto& v : C)
    if (std::fabs(v) < 1e-10) v = 0.0;
  return true;
}

}  // namespace cgtp
