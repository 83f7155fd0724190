// nbr.cpp -- periodic neighbour list by cell list, and the CSR transpose.
//
// The neighbour list reproduces exactly the brute-force definition stated in
// cgtp.h: the candidate pairs come from a cell list instead of a scan over
// all atoms and images, but every accept/reject decision evaluates the same
// FP64 expression, so the edge set and order are identical bit for bit.
// Receivers are independent: host threads take contiguous receiver ranges
// and their rows are concatenated in receiver order, so the result does not
// depend on the thread count (CGTP_HOST_THREADS overrides it; default: the
// hardware threads, one below 4096 atoms).
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <thread>
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

// Host threads for N receivers: CGTP_HOST_THREADS when set (1..256), else the
// hardware threads (at most 64), and one for small systems.
int host_threads(int64_t N) {
  if (const char* v = std::getenv("CGTP_HOST_THREADS")) {
    const int t = std::atoi(v);
    if (t >= 1) return (int)std::min<int64_t>(std::min(t, 256), std::max<int64_t>(N, 1));
  }
  if (N < 4096) return 1;
  const unsigned hw = std::thread::hardware_concurrency();
  return (int)std::max(1u, std::min(hw, 64u));
}

}  // namespace

// Cell list over the box: cells of at least the cutoff per side (at most 1024
// per axis), the atoms of each cell in index order.
struct CellList {
  int64_t nc[3], reach[3];
  double cs[3];
  std::vector<int64_t> cstart, cat, ci;
};

static cgtp_status check_and_bin(int64_t N, const double* pos, const double* box, double rc, CellList& L) {
  if (N < 0 || N >= (int64_t(1) << 31)) return fail(CGTP_ERR_SIZE, "atom count out of range");
  if (!(rc > 0.0)) return fail(CGTP_ERR_SIZE, "cutoff must be positive");
  for (int a = 0; a < 3; ++a)
    if (!(box[a] > 0.0)) return fail(CGTP_ERR_SIZE, "box lengths must be positive");
  for (int64_t i = 0; i < N; ++i)
    for (int a = 0; a < 3; ++a)
      if (!(pos[3 * i + a] >= 0.0 && pos[3 * i + a] < box[a]))
        return fail(CGTP_ERR_SIZE, "positions must lie in [0, box)");
  for (int a = 0; a < 3; ++a) {
    L.nc[a] = std::max<int64_t>(1, (int64_t)std::floor(box[a] / rc));
    L.nc[a] = std::min<int64_t>(L.nc[a], 1024);
    L.cs[a] = box[a] / (double)L.nc[a];
    L.reach[a] = (int64_t)std::floor(rc / L.cs[a]) + 1;
  }
  const int64_t ncell = L.nc[0] * L.nc[1] * L.nc[2];
  std::vector<int64_t> cell_of(N);
  L.cstart.assign(ncell + 1, 0);
  L.cat.resize(N);
  L.ci.resize(3 * N);
  for (int64_t i = 0; i < N; ++i) {
    int64_t c[3];
    for (int a = 0; a < 3; ++a) {
      c[a] = std::min<int64_t>(L.nc[a] - 1, (int64_t)(pos[3 * i + a] / L.cs[a]));
      L.ci[3 * i + a] = c[a];
    }
    cell_of[i] = (c[0] * L.nc[1] + c[1]) * L.nc[2] + c[2];
    L.cstart[cell_of[i] + 1]++;
  }
  for (int64_t c = 0; c < ncell; ++c) L.cstart[c + 1] += L.cstart[c];
  std::vector<int64_t> fill(L.cstart.begin(), L.cstart.end() - 1);
  for (int64_t i = 0; i < N; ++i) L.cat[fill[cell_of[i]]++] = i;
  return CGTP_OK;
}

// Calls fn(j, n, dx, dy, dz) for every edge i <- (j, n) of receiver i, in
// cell order (not yet sorted): the candidates of the cells within reach that
// pass the FP64 test of the definition.
template <class Fn>
static void visit_row(const CellList& L, const double* pos, const double* box, double rc2, int64_t i, Fn&& fn) {
  for (int64_t d0 = -L.reach[0]; d0 <= L.reach[0]; ++d0)
    for (int64_t d1 = -L.reach[1]; d1 <= L.reach[1]; ++d1)
      for (int64_t d2 = -L.reach[2]; d2 <= L.reach[2]; ++d2) {
        const int64_t u[3] = {L.ci[3 * i] + d0, L.ci[3 * i + 1] + d1, L.ci[3 * i + 2] + d2};
        int64_t w[3], n[3];
        for (int a = 0; a < 3; ++a) {
          n[a] = floordiv(u[a], L.nc[a]);
          w[a] = u[a] - n[a] * L.nc[a];
        }
        const int64_t c = (w[0] * L.nc[1] + w[1]) * L.nc[2] + w[2];
        for (int64_t t = L.cstart[c]; t < L.cstart[c + 1]; ++t) {
          const int64_t j = L.cat[t];
          if (j == i && n[0] == 0 && n[1] == 0 && n[2] == 0) continue;
          const double dx = (pos[3 * j] + (double)n[0] * box[0]) - pos[3 * i];
          const double dy = (pos[3 * j + 1] + (double)n[1] * box[1]) - pos[3 * i + 1];
          const double dz = (pos[3 * j + 2] + (double)n[2] * box[2]) - pos[3 * i + 2];
          const double r2 = dx * dx + dy * dy + dz * dz;
          if (r2 < rc2) fn(j, n, dx, dy, dz);
        }
      }
}

// Runs body(i0, i1) over contiguous receiver ranges on host threads; false
// when a thread could not be started or a body threw.
template <class Body>
static bool parallel_rows(int64_t N, Body&& body) {
  const int T = host_threads(N);
  std::atomic<bool> ok{true};
  auto work = [&](int t) {
    try {
      body(N * t / T, N * (t + 1) / T);
    } catch (...) {
      ok = false;
    }
  };
  std::vector<std::thread> pool;
  try {
    for (int t = 1; t < T; ++t) pool.emplace_back(work, t);
  } catch (...) {
    ok = false;
  }
  work(0);
  for (auto& th : pool) th.join();
  return ok && (int)pool.size() == T - 1;
}

cgtp_status neighbor_list_impl(int64_t N, const double* pos, const double* box, double rc,
                               int32_t* rowptr, int32_t* col, int32_t* shift, float* r,
                               int64_t* n_edges) {
  if (!pos || !box || !rowptr || !n_edges) return fail(CGTP_ERR_NULL, "null argument");
  CellList L;
  cgtp_status st;
  try {
    st = check_and_bin(N, pos, box, rc, L);
  } catch (...) {
    return fail(CGTP_ERR_OOM, "host allocation failed in the neighbour list");
  }
  if (st != CGTP_OK) return st;
  const double rc2 = rc * rc;
  // pass 1: row lengths
  std::vector<int64_t> len(N, 0);
  if (!parallel_rows(N, [&](int64_t i0, int64_t i1) {
        for (int64_t i = i0; i < i1; ++i) {
          int64_t k = 0;
          visit_row(L, pos, box, rc2, i, [&](int64_t, const int64_t*, double, double, double) { ++k; });
          len[i] = k;
        }
      }))
    return fail(CGTP_ERR_OOM, "host threads failed in the neighbour list");
  int64_t E = 0;
  for (int64_t i = 0; i < N; ++i) E += len[i];
  if (E >= (int64_t(1) << 31) - 1) return fail(CGTP_ERR_SIZE, "more than 2^31-1 edges");
  rowptr[0] = 0;
  for (int64_t i = 0; i < N; ++i) rowptr[i + 1] = (int32_t)(rowptr[i] + len[i]);
  *n_edges = E;
  if (!col) return CGTP_OK;
  // pass 2: each row sorted by (sender, image) and written at its offset
  if (!parallel_rows(N, [&](int64_t i0, int64_t i1) {
        std::vector<Cand> row;
        for (int64_t i = i0; i < i1; ++i) {
          row.clear();
          visit_row(L, pos, box, rc2, i, [&](int64_t j, const int64_t* n, double dx, double dy, double dz) {
            row.push_back({(int32_t)j, (int32_t)n[0], (int32_t)n[1], (int32_t)n[2], dx, dy, dz});
          });
          std::sort(row.begin(), row.end(), [](const Cand& a, const Cand& b) {
            return std::tie(a.j, a.nx, a.ny, a.nz) < std::tie(b.j, b.nx, b.ny, b.nz);
          });
          int64_t e = rowptr[i];
          for (const Cand& q : row) {
            col[e] = q.j;
            if (shift) {
              shift[3 * e] = q.nx;
              shift[3 * e + 1] = q.ny;
              shift[3 * e + 2] = q.nz;
            }
            if (r) {
              r[3 * e] = (float)q.dx;
              r[3 * e + 1] = (float)q.dy;
              r[3 * e + 2] = (float)q.dz;
            }
            ++e;
          }
        }
      }))
    return fail(CGTP_ERR_OOM, "host threads failed in the neighbour list");
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
