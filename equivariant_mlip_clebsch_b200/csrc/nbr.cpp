// nbr.cpp -- periodic neighbour list by cell list, and the CSR transpose.
//
// The neighbour list reproduces exactly the brute-force definition stated in
// cgtp.h: the candidate pairs come from a cell list instead of a scan over
// all atoms and images, but every accept/reject decision evaluates the same
// FP64 expression, so the edge set and order are identical bit for bit.
#include <algorithm>
#include <cmath>
#include <tuple>

#include "internal.hpp"

namespace cgtp {

namespace {

struct Cand {
  int32_t j, nx, ny, nz;
  double dx, dy, dz;
};

inline int64_t floordiv(int64_t a, int64_t b) {
  int64_t q = a / b;
  if ((a % b != 0) && ((a < 0) != (b < 0))) --q;
  return q;
}

}  // namespace

static cgtp_status neighbor_edges(int64_t N, const double* pos, const double* box, double rc,
                                  std::vector<int64_t>& start, std::vector<Cand>& edges) {
  if (N < 0 || N >= (int64_t(1) << 31)) return fail(CGTP_ERR_SIZE, "atom count out of range");
  if (!(rc > 0.0)) return fail(CGTP_ERR_SIZE, "cutoff must be positive");
  for (int a = 0; a < 3; ++a)
    if (!(box[a] > 0.0)) return fail(CGTP_ERR_SIZE, "box lengths must be positive");
  for (int64_t i = 0; i < N; ++i)
    for (int a = 0; a < 3; ++a)
      if (!(pos[3 * i + a] >= 0.0 && pos[3 * i + a] < box[a]))
        return fail(CGTP_ERR_SIZE, "positions must lie in [0, box)");
  int64_t nc[3], reach[3];
  double cs[3];
  for (int a = 0; a < 3; ++a) {
    nc[a] = std::max<int64_t>(1, (int64_t)std::floor(box[a] / rc));
    nc[a] = std::min<int64_t>(nc[a], 1024);
    cs[a] = box[a] / (double)nc[a];
    reach[a] = (int64_t)std::floor(rc / cs[a]) + 1;
  }
  const int64_t ncell = nc[0] * nc[1] * nc[2];
  std::vector<int64_t> cell_of(N), cstart(ncell + 1, 0), cat(N);
  std::vector<int64_t> ci(3 * N);
  for (int64_t i = 0; i < N; ++i) {
    int64_t c[3];
    for (int a = 0; a < 3; ++a) {
      c[a] = std::min<int64_t>(nc[a] - 1, (int64_t)(pos[3 * i + a] / cs[a]));
      ci[3 * i + a] = c[a];
    }
    cell_of[i] = (c[0] * nc[1] + c[1]) * nc[2] + c[2];
    cstart[cell_of[i] + 1]++;
  }
  for (int64_t c = 0; c < ncell; ++c) cstart[c + 1] += cstart[c];
  {
    std::vector<int64_t> fill(cstart.begin(), cstart.end() - 1);
    for (int64_t i = 0; i < N; ++i) cat[fill[cell_of[i]]++] = i;
  }
  const double rc2 = rc * rc;
  start.assign(N + 1, 0);
  edges.clear();
  std::vector<Cand> row;
  for (int64_t i = 0; i < N; ++i) {
    row.clear();
    for (int64_t d0 = -reach[0]; d0 <= reach[0]; ++d0)
      for (int64_t d1 = -reach[1]; d1 <= reach[1]; ++d1)
        for (int64_t d2 = -reach[2]; d2 <= reach[2]; ++d2) {
          const int64_t u[3] = {ci[3 * i] + d0, ci[3 * i + 1] + d1, ci[3 * i + 2] + d2};
          int64_t w[3], n[3];
          for (int a = 0; a < 3; ++a) {
            n[a] = floordiv(u[a], nc[a]);
            w[a] = u[a] - n[a] * nc[a];
          }
          const int64_t c = (w[0] * nc[1] + w[1]) * nc[2] + w[2];
          for (int64_t t = cstart[c]; t < cstart[c + 1]; ++t) {
            const int64_t j = cat[t];
            if (j == i && n[0] == 0 && n[1] == 0 && n[2] == 0) continue;
            const double dx = (pos[3 * j] + (double)n[0] * box[0]) - pos[3 * i];
            const double dy = (pos[3 * j + 1] + (double)n[1] * box[1]) - pos[3 * i + 1];
            const double dz = (pos[3 * j + 2] + (double)n[2] * box[2]) - pos[3 * i + 2];
            const double d2 = dx * dx + dy * dy + dz * dz;
            if (d2 < rc2) row.push_back({(int32_t)j, (int32_t)n[0], (int32_t)n[1], (int32_t)n[2], dx, dy, dz});
          }
        }
    std::sort(row.begin(), row.end(), [](const Cand& a, const Cand& b) {
      return std::tie(a.j, a.nx, a.ny, a.nz) < std::tie(b.j, b.nx, b.ny, b.nz);
    });
    edges.insert(edges.end(), row.begin(), row.end());
    start[i + 1] = (int64_t)edges.size();
  }
  if ((int64_t)edges.size() >= (int64_t(1) << 31) - 1)
    return fail(CGTP_ERR_SIZE, "more than 2^31-1 edges");
  return CGTP_OK;
}

cgtp_status neighbor_list_impl(int64_t N, const double* pos, const double* box, double rc,
                               int32_t* rowptr, int32_t* col, int32_t* shift, float* r,
                               int64_t* n_edges) {
  if (!pos || !box || !rowptr || !n_edges) return fail(CGTP_ERR_NULL, "null argument");
  std::vector<int64_t> start;
  std::vector<Cand> edges;
  cgtp_status st = neighbor_edges(N, pos, box, rc, start, edges);
  if (st != CGTP_OK) return st;
  for (int64_t i = 0; i <= N; ++i) rowptr[i] = (int32_t)start[i];
  *n_edges = (int64_t)edges.size();
  if (!col) return CGTP_OK;
  for (size_t e = 0; e < edges.size(); ++e) {
    col[e] = edges[e].j;
    if (shift) {
      shift[3 * e] = edges[e].nx;
      shift[3 * e + 1] = edges[e].ny;
      shift[3 * e + 2] = edges[e].nz;
    }
    if (r) {
      r[3 * e] = (float)edges[e].dx;
      r[3 * e + 1] = (float)edges[e].dy;
      r[3 * e + 2] = (float)edges[e].dz;
    }
  }
  return CGTP_OK;
}

cgtp_status check_csr(int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                      const int32_t* col) {
  if (rowptr[0] != 0 || rowptr[n_recv] != E) return fail(CGTP_ERR_INVALID_CSR, "rowptr ends mismatch");
  for (int64_t i = 0; i < n_recv; ++i)
    if (rowptr[i + 1] < rowptr[i]) return fail(CGTP_ERR_INVALID_CSR, "rowptr not monotone");
  for (int64_t e = 0; e < E; ++e)
    if (col[e] < 0 || col[e] >= n_send) return fail(CGTP_ERR_INVALID_CSR, "col out of range");
  return CGTP_OK;
}

cgtp_status csr_transpose_impl(int64_t n_recv, int64_t n_send, int64_t E, const int32_t* rowptr,
                               const int32_t* col, int32_t* rowptr_T, int32_t* perm_T) {
  if (!rowptr || !rowptr_T || (E > 0 && (!col || !perm_T))) return fail(CGTP_ERR_NULL, "null argument");
  if (n_recv < 0 || n_send < 0 || E < 0 || E >= (int64_t(1) << 31) - 1)
    return fail(CGTP_ERR_SIZE, "sizes out of range");
  cgtp_status st = check_csr(n_recv, n_send, E, rowptr, col);
  if (st != CGTP_OK) return st;
  std::vector<int64_t> cnt(n_send + 1, 0);
  for (int64_t e = 0; e < E; ++e) cnt[col[e] + 1]++;
  for (int64_t j = 0; j < n_send; ++j) cnt[j + 1] += cnt[j];
  for (int64_t j = 0; j <= n_send; ++j) rowptr_T[j] = (int32_t)cnt[j];
  for (int64_t e = 0; e < E; ++e) perm_T[cnt[col[e]]++] = (int32_t)e;
  return CGTP_OK;
}

}  // namespace cgtp
