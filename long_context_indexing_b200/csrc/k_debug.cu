// k_debug.cu -- the checks the library runs when the environment variable
// LSA_DEBUG=1 is set at load time (a debugging aid, not part of the method).
//
// They validate, at the ABI boundary, the data every gather of the hot path
// reads, so that a corrupted index or selection is reported (LSA_ERR_INTERNAL,
// with what and where) before a kernel consumes it:
//   index     (debug_index_kernel, a CTA per closed block and sequence, plus
//             one for the open block): the block's CSR offsets start at its
//             first pooled group, end at its last, never decrease; every
//             member lies in the block, members ascend inside a bucket and
//             each one's k-means assignment names that bucket (so the members
//             are a permutation of the block); open-block entries are -1 or a
//             closed bucket id;
//   selection (debug_gather_kernel, a warp per row): 0 <= count <= s_max and
//             every listed index inside [0, T_cap); for selections the library
//             made, the row's layout: sinks 0 .. n_s-1 first, the window
//             max(pos-W+1, n_s) .. pos last, every long-range key in between
//             inside [S, pos - W] (and ascending for the per-key indexer).
// A violation is recorded in a library-owned device word (first one wins:
// kind, sequence or row, place, value); the host reads it after a stream
// synchronisation and clears it.  The word is one per device: checks that
// run at the same time on several streams or threads share it, so a debug
// session serialises its calls.  No check traps or faults: a check that finds
// a bad offset skips the reads it would have guarded.
#include "lsa_internal.cuh"

namespace lsa {

__device__ uint32_t g_dbg[4];

__device__ __forceinline__ void dbg_report(uint32_t kind, int64_t who, int64_t where, int64_t value)
{
    if (atomicCAS(&g_dbg[0], 0u, kind) == 0u) {
        g_dbg[1] = (uint32_t)who;
        g_dbg[2] = (uint32_t)where;
        g_dbg[3] = (uint32_t)value;
    }
}

constexpr int DBG_THREADS = 256;

__global__ void __launch_bounds__(DBG_THREADS) debug_index_kernel(IndexView ix, int64_t n_blk)
{
    __shared__ int ok;
    const int64_t b = blockIdx.y;
    const int64_t blk = blockIdx.x;
    const int k = ix.k, G = ix.G;
    if (blk == n_blk) {
        // the open block: entries are -1 or closed bucket ids (before the
        // first closed block the list is not read)
        if (n_blk == 0) return;
        const int32_t* open = ix.open_bucket + b * G;
        for (int o = threadIdx.x; o < G; o += DBG_THREADS) {
            const int32_t g = open[o];
            if (g < -1 || g >= n_blk * k) dbg_report(DBG_OPEN, b, o, g);
        }
        return;
    }
    const int32_t* off = ix.offsets + b * (ix.NBK + 1) + blk * k;
    const int32_t* mem = ix.members + b * ix.NP;
    const int16_t* as = ix.assign + b * ix.NP;
    const int64_t jb = blk * G;
    if (threadIdx.x == 0) {
        ok = 1;
        if (off[0] != jb || off[k] != jb + G) {
            dbg_report(DBG_OFFSETS, b, blk * k, off[0] != jb ? off[0] : off[k]);
            ok = 0;
        }
    }
    __syncthreads();
    for (int m = threadIdx.x; m < k; m += DBG_THREADS)
        if (off[m] > off[m + 1] || off[m] < jb || off[m + 1] > jb + G) {
            dbg_report(DBG_OFFSETS, b, blk * k + m, off[m]);
            ok = 0;
        }
    __syncthreads();
    if (!ok) return;                                 // the member reads below need sane offsets
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int m = warp; m < k; m += DBG_THREADS / 32) {
        const int32_t o0 = off[m], o1 = off[m + 1];
        for (int32_t x = o0 + lane; x < o1; x += 32) {
            const int32_t v = mem[x];
            if (v < jb || v >= jb + G) {
                dbg_report(DBG_MEMBER, b, x, v);
                continue;
            }
            if (x > o0 && mem[x - 1] >= v) dbg_report(DBG_ORDER, b, x, v);
            if (as[v] != m) dbg_report(DBG_ASSIGN, b, v, as[v]);
        }
    }
}

// mode 0: bounds only; 1: a selection's layout; 2: layout, long-range keys ascending.
__global__ void __launch_bounds__(DBG_THREADS) debug_gather_kernel(
    const int32_t* indices, const int32_t* counts, int64_t rows, int s_max, int64_t T_cap,
    PosSrc pos, int64_t Nq, int W, int S, int mode)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (DBG_THREADS / 32) + (threadIdx.x >> 5);
    if (row >= rows) return;                          // warp-uniform
    const int n = counts[row];
    if (n < 0 || n > s_max) {
        if (lane == 0) dbg_report(DBG_COUNT, row, 0, n);
        return;
    }
    const int32_t* in = indices + row * (int64_t)s_max;
    int64_t n_s = 0, w0 = 0, n_w = 0, p = T_cap - 1;
    if (mode > 0) {
        p = pos.at(row / Nq, Nq, row % Nq);
        n_s = (p + 1 < S) ? p + 1 : S;
        w0 = (p - W + 1 > n_s) ? p - W + 1 : n_s;
        n_w = p - w0 + 1;
        if (n_s + n_w > n) {
            if (lane == 0) dbg_report(DBG_COUNT, row, 1, n);
            return;
        }
    }
    for (int j = lane; j < n; j += 32) {
        const int32_t t = in[j];
        if (t < 0 || t >= T_cap) {
            dbg_report(DBG_INDEX, row, j, t);
        } else if (mode > 0) {
            bool good;
            if (j < n_s) good = t == j;
            else if (j >= n - n_w) good = t == w0 + (j - (n - n_w));
            else good = t >= S && t <= p - W && (mode < 2 || j == n_s || in[j - 1] < t);
            if (!good) dbg_report(t > p ? DBG_CAUSAL : DBG_LAYOUT, row, j, t);
        }
    }
}

bool debug_enabled()
{
    static const bool on = [] {
        const char* e = getenv("LSA_DEBUG");
        return e && e[0] == '1' && e[1] == 0;
    }();
    return on;
}

// Runs when the stream can be synchronised (not under capture): returns the
// recorded violation (kind 0 = none) and clears it.
static cudaError_t dbg_collect(cudaStream_t st, uint32_t out[4])
{
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_dbg, 4 * sizeof(uint32_t), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e == cudaSuccess && out[0] != 0u) {
        static const uint32_t zero[4] = {0u, 0u, 0u, 0u};
        e = cudaMemcpyToSymbolAsync(g_dbg, zero, sizeof(zero), 0, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    }
    return e;
}

static bool capturing(cudaStream_t st)
{
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    return cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs != cudaStreamCaptureStatusNone;
}

cudaError_t debug_check_index(const IndexView& ix, int64_t n_blk, cudaStream_t st, uint32_t out[4])
{
    out[0] = 0u;
    if (capturing(st)) return cudaSuccess;
    debug_index_kernel<<<dim3((unsigned)(n_blk + 1), (unsigned)ix.B), DBG_THREADS, 0, st>>>(ix, n_blk);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = dbg_collect(st, out);
    return e;
}

cudaError_t debug_check_gather(const int32_t* indices, const int32_t* counts, int64_t rows,
                               int s_max, int64_t T_cap, PosSrc pos, int64_t Nq, int W, int S,
                               int mode, cudaStream_t st, uint32_t out[4])
{
    out[0] = 0u;
    if (rows <= 0 || capturing(st)) return cudaSuccess;
    const int64_t grid = (rows + DBG_THREADS / 32 - 1) / (DBG_THREADS / 32);
    debug_gather_kernel<<<(unsigned)grid, DBG_THREADS, 0, st>>>(indices, counts, rows, s_max, T_cap,
                                                                pos, Nq, W, S, mode);
    note_launch();
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = dbg_collect(st, out);
    return e;
}

}  // namespace lsa
