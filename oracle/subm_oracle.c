/*
 * CPU oracle for submanifold sparse 3-D convolution (SubMConv3d).
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
 * baseline leg may load this file's library.  It shares no code with the CUDA
 * path and the CUDA path never calls it.
 *
 * What it computes (the plain definition, no blocking or reordering):
 *
 *   out[i] = bias + sum over offsets d in {-1,0,1}^3 with p_i + d active of
 *            W[k(d)]^T x[index of p_i + d]
 *
 * Sources on the pages:
 *   - lato.2_mrp_mlx README, "Status": SubMConv3d with k=3 and k=1.
 *   - lato.2_mrp_mlx README, "Correctness": the reference is a naive
 *     dictionary lookup with a per-voxel loop; the implemented orientation
 *     gathers feats[c+d] (cross-correlation).  We follow c+d.
 *   - lato.2_mrp_mlx README, "The scope, once measured": stride 1 and
 *     padding None, i.e. outputs exist only at the input's active sites.
 *   - pixal3d_mrp_mlx README, "Status": kernels are laid out [K^3, in, out].
 *   - trellis-mac article (Japanese), "sparse 3D convolution -> gather-scatter":
 *     a map of active voxel coordinates is built first, then probed per
 *     kernel offset.
 *
 * Orientation option: the same README section says the upstream orientation
 * is unverified and that its --flip-kernel switch builds the alternative, which
 * gathers feats[c-d]; oracle_neighbor_map_oriented with flip = 1 computes that
 * map (neighbour at p_i - d_k).
 *
 * Readings where the pages are silent:
 *   - offset order: k = (dx+1)*9 + (dy+1)*3 + (dz+1), dx slowest, matching
 *     coordinate columns (x, y, z); the centre is k = 13.  For k=1, one offset.
 *   - a neighbour must share the batch index; neighbours outside [0, extent)
 *     are holes.
 *   - a coordinate outside [0, extent) or a batch index outside [0, 65535] is
 *     an error (ORACLE_COORD_RANGE); a repeated (b,x,y,z) is an error
 *     (ORACLE_DUPLICATE).
 *   - accumulation in fp64 from the exact input values.
 *
 * The "dictionary" is a sorted array of (key, row) pairs searched with the C
 * library's bsearch; the key packs (b, x, y, z) in 16 bits each.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum {
    ORACLE_OK = 0,
    ORACLE_INVALID_ARG = 1,
    ORACLE_COORD_RANGE = 3,
    ORACLE_DUPLICATE = 4,
    ORACLE_OOM = 6,
};

typedef struct {
    uint64_t key;
    int64_t row;
} entry_t;

static uint64_t pack_key(int64_t b, int64_t x, int64_t y, int64_t z) {
    return ((uint64_t)b << 48) | ((uint64_t)x << 32) | ((uint64_t)y << 16) | (uint64_t)z;
}

static int cmp_entry(const void* a, const void* b) {
    uint64_t ka = ((const entry_t*)a)->key, kb = ((const entry_t*)b)->key;
    return (ka > kb) - (ka < kb);
}

/* Neighbour map: nbr[i * K^3 + k] = row of the active voxel at p_i + s d_k, else
 * -1, with s = +1 (flip = 0) or s = -1 (flip = 1).
 * coords is int32 [n, 4] = (b, x, y, z); extent = (X, Y, Z), each in [1, 65535].
 * Returns ORACLE_OK or an error code; on error nbr is left unspecified. */
int oracle_neighbor_map_oriented(const int32_t* coords, int64_t n, const int32_t* extent,
                                 int32_t kernel_size, int32_t flip, int32_t* nbr) {
    if (n < 0 || (n > 0 && (!coords || !nbr)) || !extent) return ORACLE_INVALID_ARG;
    if (kernel_size != 1 && kernel_size != 3) return ORACLE_INVALID_ARG;
    for (int a = 0; a < 3; ++a)
        if (extent[a] < 1 || extent[a] > 65535) return ORACLE_INVALID_ARG;
    if (n == 0) return ORACLE_OK;

    for (int64_t i = 0; i < n; ++i) {
        const int32_t* c = coords + 4 * i;
        if (c[0] < 0 || c[0] > 65535) return ORACLE_COORD_RANGE;
        for (int a = 0; a < 3; ++a)
            if (c[1 + a] < 0 || c[1 + a] >= extent[a]) return ORACLE_COORD_RANGE;
    }

    entry_t* dict = (entry_t*)malloc((size_t)n * sizeof(entry_t));
    if (!dict) return ORACLE_OOM;
    for (int64_t i = 0; i < n; ++i) {
        const int32_t* c = coords + 4 * i;
        dict[i].key = pack_key(c[0], c[1], c[2], c[3]);
        dict[i].row = i;
    }
    qsort(dict, (size_t)n, sizeof(entry_t), cmp_entry);
    for (int64_t i = 1; i < n; ++i) {
        if (dict[i].key == dict[i - 1].key) {
            free(dict);
            return ORACLE_DUPLICATE;
        }
    }

    const int kvol = kernel_size * kernel_size * kernel_size;
    const int r = kernel_size / 2;
    const int s = flip ? -1 : 1;
    for (int64_t i = 0; i < n; ++i) {
        const int32_t* c = coords + 4 * i;
        int k = 0;
        for (int dx = -r; dx <= r; ++dx)
            for (int dy = -r; dy <= r; ++dy)
                for (int dz = -r; dz <= r; ++dz, ++k) {
                    int64_t x = (int64_t)c[1] + s * dx, y = (int64_t)c[2] + s * dy, z = (int64_t)c[3] + s * dz;
                    int32_t found = -1;
                    if (x >= 0 && x < extent[0] && y >= 0 && y < extent[1] && z >= 0 && z < extent[2]) {
                        entry_t probe;
                        probe.key = pack_key(c[0], x, y, z);
                        probe.row = 0;
                        const entry_t* hit = (const entry_t*)bsearch(&probe, dict, (size_t)n,
                                                                     sizeof(entry_t), cmp_entry);
                        if (hit) found = (int32_t)hit->row;
                    }
                    nbr[i * kvol + k] = found;
                }
    }
    free(dict);
    return ORACLE_OK;
}

int oracle_neighbor_map(const int32_t* coords, int64_t n, const int32_t* extent,
                        int32_t kernel_size, int32_t* nbr) {
    return oracle_neighbor_map_oriented(coords, n, extent, kernel_size, 0, nbr);
}

/* Forward pass in fp64 for the output rows listed in `rows` (all rows when rows
 * is NULL; then nrows must equal n).  out is [nrows, cout] in the order of rows.
 * x is [n, cin], w is [kvol, cin, cout], bias is [cout] or NULL. */
int oracle_forward_f64(const int32_t* nbr, int64_t n, int32_t kvol,
                       const double* x, int32_t cin,
                       const double* w, const double* bias, int32_t cout,
                       const int64_t* rows, int64_t nrows, double* out) {
    if (n < 0 || nrows < 0 || cin < 1 || cout < 1 || (kvol != 1 && kvol != 27)) return ORACLE_INVALID_ARG;
    if (!rows && nrows != n) return ORACLE_INVALID_ARG;
    if (nrows > 0 && (!nbr || !x || !w || !out)) return ORACLE_INVALID_ARG;
    for (int64_t t = 0; t < nrows; ++t) {
        int64_t i = rows ? rows[t] : t;
        if (i < 0 || i >= n) return ORACLE_INVALID_ARG;
        double* acc = out + t * cout;
        for (int32_t co = 0; co < cout; ++co) acc[co] = bias ? bias[co] : 0.0;
        for (int32_t k = 0; k < kvol; ++k) {
            int32_t j = nbr[i * kvol + k];
            if (j < 0) continue;
            const double* xj = x + (int64_t)j * cin;
            const double* wk = w + (int64_t)k * cin * cout;
            for (int32_t ci = 0; ci < cin; ++ci) {
                const double xv = xj[ci];
                const double* wrow = wk + (int64_t)ci * cout;
                for (int32_t co = 0; co < cout; ++co) acc[co] += xv * wrow[co];
            }
        }
    }
    return ORACLE_OK;
}
