// CPU oracle for the submanifold 3x3x3 sparse convolution (SubMConv3d).
//
// TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the CPU-baseline
// leg of the benchmark may load this library.  It shares no code, header,
// table or helper with the CUDA path in sparse_voxel_conv_b200/.
//
// It is the plain definition of the op written out, slow on purpose:
//   * the coordinate set is a std::map keyed by the (b, z, y, x) tuple
//     ("sorted-key indice map ... 27 lookups/voxel", lato.2_mrp_mlx, commit
//     97dcdfb54a message);
//   * the forward is a per-voxel, per-offset loop accumulated in fp64
//     ("an independent naive reference ... shares no indexing code", same
//     commit message; "Conventions" in that page's CLAUDE.md notes).
//
// Conventions (stated readings of the pages):
//   * offsets are ordered kz-major: k = 9*(dz+1) + 3*(dy+1) + (dx+1), the
//     order of spconv's KRSC weight [Cout, kz, ky, kx, Cin] (lato.2_mrp_mlx
//     CLAUDE.md, "Key facts");
//   * correlation: out[i] = sum_k W[:, k, :] . x[voxel at p_i + d_k]; with
//     flip the mirrored slice W[:, 26-k, :] is used instead (the
//     --flip-kernel mirror of the same commit message and the "Unresolved"
//     section of the notes);
//   * a neighbour outside [0, grid_dim)^3 or absent from the set is -1;
//     voxels of different batch elements are never neighbours.
//
// Build: g++ -O2 -fopenmp -shared -fPIC subm3d_oracle.cpp -o liboracle.so

#include <array>
#include <cmath>
#include <cstdint>
#include <map>
#include <omp.h>

namespace {

using Key = std::array<int32_t, 4>;   // (b, z, y, x)

enum { ORACLE_OK = 0, ORACLE_RANGE = 2, ORACLE_DUPLICATE = 3 };

}  // namespace

extern "C" {

// Number of OpenMP threads the oracle's parallel loops use.
int oracle_num_threads(void) { return omp_get_max_threads(); }

// Neighbour map: nbr[i*27 + k] = row of the voxel at p_i + d_k, or -1.
// Returns 0, or 2 when a coordinate lies outside [0,batch) x [0,grid_dim)^3,
// or 3 when a coordinate occurs twice.  nbr is left unspecified on error.
int oracle_build_map(const int32_t* coords, int64_t n, int32_t grid_dim,
                     int32_t batch, int32_t* nbr) {
  std::map<Key, int64_t> rows;
  for (int64_t i = 0; i < n; ++i) {
    const int32_t* c = coords + 4 * i;
    if (c[0] < 0 || c[0] >= batch) return ORACLE_RANGE;
    for (int a = 1; a < 4; ++a)
      if (c[a] < 0 || c[a] >= grid_dim) return ORACLE_RANGE;
    Key key = {c[0], c[1], c[2], c[3]};
    if (!rows.emplace(key, i).second) return ORACLE_DUPLICATE;
  }
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const int32_t* c = coords + 4 * i;
    int k = 0;
    for (int dz = -1; dz <= 1; ++dz)
      for (int dy = -1; dy <= 1; ++dy)
        for (int dx = -1; dx <= 1; ++dx, ++k) {
          Key q = {c[0], c[1] + dz, c[2] + dy, c[3] + dx};
          auto it = rows.find(q);
          nbr[i * 27 + k] = (it == rows.end()) ? -1 : (int32_t)it->second;
        }
  }
  return ORACLE_OK;
}

// Forward, fp64: for each requested output row r (rows == nullptr means all
// rows 0..n-1, else rows[0..n_rows)):
//   out[r_pos*cout + o] = sum_{k=0}^{26} sum_{c} Wf[o][k][c] * x[nbr[r][k]][c]
// over the k with nbr[r][k] != -1, where Wf[o][k] = W[o][k] (correlation) or
// W[o][26-k] (flip).  x is [n_src, cin] and W is [cout, 27, cin], both fp64.
void oracle_forward(const int32_t* nbr, const double* x, const double* w,
                    int32_t cin, int32_t cout, int32_t flip,
                    const int64_t* rows, int64_t n_rows, double* out) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t p = 0; p < n_rows; ++p) {
    const int64_t r = rows ? rows[p] : p;
    double* o_row = out + p * cout;
    for (int32_t o = 0; o < cout; ++o) o_row[o] = 0.0;
    for (int k = 0; k < 27; ++k) {
      const int32_t j = nbr[r * 27 + k];
      if (j < 0) continue;
      const int kw = flip ? 26 - k : k;
      const double* xj = x + (int64_t)j * cin;
      for (int32_t o = 0; o < cout; ++o) {
        const double* wk = w + ((int64_t)o * 27 + kw) * cin;
        double s = 0.0;
        for (int32_t c = 0; c < cin; ++c) s += wk[c] * xj[c];
        o_row[o] += s;
      }
    }
  }
}

// Gradient with respect to the input features, fp64, by scattering each term of
// the forward back to its source row:
//   dx[j][c] += sum_o Wf[o][k][c] * dy[i][o]   for every (i, k) with nbr[i][k] = j.
// dy is [n, cout], W is [cout, 27, cin], dx is [n, cin] (overwritten).  Serial
// in i (the scatter targets collide); n is small in the tests that call it.
void oracle_backward_data(const int32_t* nbr, int64_t n, const double* dy, const double* w,
                          int32_t cin, int32_t cout, int32_t flip, double* dx) {
  for (int64_t e = 0; e < n * cin; ++e) dx[e] = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    for (int k = 0; k < 27; ++k) {
      const int32_t j = nbr[i * 27 + k];
      if (j < 0) continue;
      const int kw = flip ? 26 - k : k;
      for (int32_t o = 0; o < cout; ++o) {
        const double g = dy[i * cout + o];
        const double* wk = w + ((int64_t)o * 27 + kw) * cin;
        for (int32_t c = 0; c < cin; ++c) dx[(int64_t)j * cin + c] += wk[c] * g;
      }
    }
  }
}

// Gradient with respect to the weight, fp64:
//   dW[o][kw][c] += dy[i][o] * x[nbr[i][k]][c]   for every (i, k), nbr[i][k] != -1,
// kw = k (correlation) or 26 - k (flip).  dW is [cout, 27, cin] (overwritten).
// Parallel over the output channel o (each thread owns its rows of dW).
void oracle_backward_weight(const int32_t* nbr, int64_t n, const double* x, const double* dy,
                            int32_t cin, int32_t cout, int32_t flip, double* dw) {
#pragma omp parallel for schedule(static)
  for (int32_t o = 0; o < cout; ++o) {
    double* dwo = dw + (int64_t)o * 27 * cin;
    for (int64_t e = 0; e < 27 * (int64_t)cin; ++e) dwo[e] = 0.0;
    for (int64_t i = 0; i < n; ++i) {
      const double g = dy[i * cout + o];
      for (int k = 0; k < 27; ++k) {
        const int32_t j = nbr[i * 27 + k];
        if (j < 0) continue;
        const int kw = flip ? 26 - k : k;
        const double* xj = x + (int64_t)j * cin;
        double* d = dwo + (int64_t)kw * cin;
        for (int32_t c = 0; c < cin; ++c) d[c] += g * xj[c];
      }
    }
  }
}

// Exact-erf GELU in place: v <- 0.5 * v * (1 + erf(v / sqrt(2))).
void oracle_gelu(double* v, int64_t n) {
  for (int64_t i = 0; i < n; ++i) v[i] = 0.5 * v[i] * (1.0 + std::erf(v[i] / std::sqrt(2.0)));
}

// SiLU in place: v <- v * sigmoid(v) = v / (1 + exp(-v)).
void oracle_silu(double* v, int64_t n) {
  for (int64_t i = 0; i < n; ++i) v[i] = v[i] / (1.0 + std::exp(-v[i]));
}

// Round in place to the nearest bfloat16 value, ties to even.  bfloat16 keeps
// 8 significant bits and float32's exponent range (normal numbers down to
// 2^-126, subnormal spacing 2^-133, largest finite (2 - 2^-7) * 2^127).
void oracle_round_bf16(double* v, int64_t n) {
  for (int64_t i = 0; i < n; ++i) {
    double a = v[i];
    if (a == 0.0 || !std::isfinite(a)) continue;
    int e;
    std::frexp(a, &e);                 // a = m * 2^e, 0.5 <= |m| < 1
    int q = e - 8;                     // spacing of 8-bit significands at this binade
    if (q < -133) q = -133;            // subnormal range keeps a fixed spacing
    double r = std::ldexp(std::nearbyint(std::ldexp(a, -q)), q);  // nearbyint: ties-to-even
    const double max_bf16 = std::ldexp(255.0, 120);               // (2 - 2^-7) * 2^127
    if (std::fabs(r) > max_bf16) r = std::copysign(INFINITY, a);
    v[i] = r;
  }
}

}  // extern "C"
