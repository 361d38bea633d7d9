// schedule.cu -- block levels -> token levels -> per-step ascending lists of
// due tokens for the whole interleaved schedule (Jano pages: nl technical
// summary, Methodologie 2: warm-up, Level 1 rarely, Level 2 intermittently,
// Level 3 every step, cool-down; zh 2.2 item 2).
//
// Because a step's due set is a union of whole levels, the position of a
// token in step s's list is
//     offsets[s] + sum over due levels l of (tokens of level l in earlier tiles)
//                + (due tokens before it inside its tile),
// so no step has to wait on another and no tile on another:
//   1. count   one CTA per 1024-token tile: token level (from the block map)
//              stored to scratch, per-level counts of the tile via warp ballots;
//   2. write   one CTA per (tile, chunk of steps): its per-level prefix over
//              the earlier tiles and the level totals by a block reduction
//              over the tile counts, the step offsets in closed form from
//              those totals, the tile's tokens ranked once in each of the four
//              possible due sets (ballot + popc + one warp scan per set), then
//              ascending stores of the due ids of the chunk's steps.  The
//              chunks spread the stores of the 50 steps over every SM.  It is
//              launched as a programmatic dependent of the count pass: its
//              CTAs become resident while the count pass runs and wait
//              (griddepcontrol.wait) for its results before reading them.
// Scratch (caller-provided): token levels [n_tokens] u8 and tile counts
// [3][n_tiles] int32, each part 16-byte aligned.
#include <algorithm>

#include "jano_common.cuh"

namespace jano {
namespace {

constexpr int kTile = 1024;       // tokens per tile == threads per CTA

struct Geo {
    int TF, TH, TW;               // token grid
    int pf, ph, pw;
    int nBh, nBw;
    int bf, bh, bw;
    int n_blocks;
};

struct Ws {
    uint8_t* tok;                 // [n_tokens]
    int* cnt;                     // [3][n_tiles]   (level-1 index)
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

Ws carve(void* base, long long n_tokens, int n_tiles) {
    char* p = static_cast<char*>(base);
    Ws w;
    w.tok = reinterpret_cast<uint8_t*>(p);
    p += align16((size_t)n_tokens);
    w.cnt = reinterpret_cast<int*>(p);
    return w;
}

__device__ __forceinline__ bool level_due(int lv, bool due2, bool due1) {
    return lv == 3 || (lv == 2 && due2) || (lv == 1 && due1);
}

__device__ __forceinline__ void step_due(int s, const jano_sched_cfg& c, bool& due2, bool& due1) {
    const bool full = s < c.warmup || s >= c.T - c.cooldown;
    const int j = s - c.warmup;
    due2 = full || ((j + 1) % c.period_moderate == 0);
    due1 = full || ((j + 1) % c.period_static == 0);
}

__global__ void __launch_bounds__(kTile)
count_kernel(const uint8_t* __restrict__ block_levels, Geo g, int n_tokens,
             uint8_t* __restrict__ token_levels, Ws ws, int n_tiles, int* err) {
    // the write pass may be scheduled now; it reads nothing of ours before
    // this grid has completed (griddepcontrol.wait)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ int wc[3][32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.x * kTile + tid;
    int lv = 0;
    if (t < n_tokens) {
        const int tw = t % g.TW;
        const int r = t / g.TW;
        const int th = r % g.TH;
        const int tf = r / g.TH;
        const int b = ((tf * g.pf) / g.bf * g.nBh + (th * g.ph) / g.bh) * g.nBw + (tw * g.pw) / g.bw;
        lv = __ldg(block_levels + b);
        if (lv < 1 || lv > 3) {
            raise_error(err, JANO_EINDEX);
            lv = 1;
        }
        ws.tok[t] = (uint8_t)lv;
        if (token_levels) token_levels[t] = (uint8_t)lv;
    }
#pragma unroll
    for (int l = 0; l < 3; ++l) {
        const unsigned b = __ballot_sync(0xFFFFFFFFu, lv == l + 1);
        if (lane == 0) wc[l][warp] = __popc(b);
    }
    __syncthreads();
    if (warp < 3) {
        int v = wc[warp][lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0) ws.cnt[warp * n_tiles + blockIdx.x] = v;
    }
}

// Due tokens of every step before step s, in closed form from the level
// totals n1, n2, n3: each step lists Level 3; Level 2 when due2, Level 1 when
// due1.  D(s, p) counts the steps s' < s in which a level of period p is due
// (full steps count too).
__device__ __forceinline__ long long due_before(int s, int p, const jano_sched_cfg& c) {
    const int w = c.warmup, e = c.T - c.cooldown;        // interleaved steps are [w, e)
    if (s <= w) return s;
    const int si = min(s, e);
    long long d = w + (si - w) / p;                      // j + 1 = 1 .. si - w, multiples of p
    if (s > e) d += s - e;
    return d;
}

__device__ __forceinline__ long long offset_of(int s, const jano_sched_cfg& c, const int (&tot)[3]) {
    return (long long)s * tot[2] + due_before(s, c.period_moderate, c) * tot[1] +
           due_before(s, c.period_static, c) * tot[0];
}

// The due set of a step is one of four unions of levels: {3}, {3,2}, {3,1},
// {3,2,1} (set id = due2 | due1 << 1).  One CTA per tile: it forms the
// tile's per-level prefix over the earlier tiles and the level totals from
// the count pass (a block reduction over the tile counts, no separate scan
// launch), ranks the tile's tokens once in each of the four sets (ballots +
// one warp scan per set) and stores the tile's part of every step's list;
// the first CTA also writes offsets[].
__global__ void __launch_bounds__(kTile)
write_kernel(Ws ws, int n_tokens, int n_tiles, jano_sched_cfg c,
             int32_t* __restrict__ offsets, int32_t* __restrict__ idx) {
    __shared__ int wc[4][32];
    __shared__ int wpre[4][32];
    __shared__ int red[6][32];
    __shared__ int s_pre[3], s_tot[3];
    constexpr int kStepChunk = 1024;
    __shared__ long long s_base[kStepChunk];     // offsets of a chunk of steps
    __shared__ unsigned char s_set[kStepChunk];  // their due sets
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tile = blockIdx.x;
    // this CTA's steps: chunk blockIdx.y of gridDim.y
    const int s_lo = (int)((long long)c.T * blockIdx.y / gridDim.y);
    const int s_hi = (int)((long long)c.T * (blockIdx.y + 1) / gridDim.y);
    // the count pass's token levels and tile counts are complete and visible after this
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- per-level prefix over earlier tiles and totals over all tiles
    int pre[3] = {0, 0, 0}, tot[3] = {0, 0, 0};
    for (int i = tid; i < n_tiles; i += kTile) {
#pragma unroll
        for (int l = 0; l < 3; ++l) {
            const int v = ws.cnt[l * n_tiles + i];
            tot[l] += v;
            if (i < tile) pre[l] += v;
        }
    }
#pragma unroll
    for (int l = 0; l < 3; ++l) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            pre[l] += __shfl_xor_sync(0xFFFFFFFFu, pre[l], o);
            tot[l] += __shfl_xor_sync(0xFFFFFFFFu, tot[l], o);
        }
        if (lane == 0) { red[l][warp] = pre[l]; red[3 + l][warp] = tot[l]; }
    }

    // ---- ranks of the tile's tokens in the four due sets
    const int t = tile * kTile + tid;
    const int lv = t < n_tokens ? ws.tok[t] : 0;
    const unsigned lt = (1u << lane) - 1u;
    bool in[4];
    int rank[4];
#pragma unroll
    for (int set = 0; set < 4; ++set) {
        in[set] = t < n_tokens && level_due(lv, set & 1, (set >> 1) & 1);
        const unsigned b = __ballot_sync(0xFFFFFFFFu, in[set]);
        rank[set] = __popc(b & lt);
        if (lane == 0) wc[set][warp] = __popc(b);
    }
    __syncthreads();
    if (warp < 6) {
        int v = red[warp][lane];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0) {
            if (warp < 3) s_pre[warp] = v;
            else s_tot[warp - 3] = v;
        }
    } else if (warp < 10) {
        const int set = warp - 6;
        const int v = wc[set][lane];
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        wpre[set][lane] = incl - v;
    }
    __syncthreads();
    const int total[3] = {s_tot[0], s_tot[1], s_tot[2]};
    // position of this token inside step lists of each set, less the step's offset
    int pos[4];
#pragma unroll
    for (int set = 0; set < 4; ++set)
        pos[set] = s_pre[2] + ((set & 1) ? s_pre[1] : 0) + ((set & 2) ? s_pre[0] : 0) +
                   wpre[set][warp] + rank[set];
    if (tile == 0 && s_lo == 0 && tid == 0) offsets[0] = 0;

    // ---- this tile's part of the chunk's steps, staged kStepChunk at a time
    for (int s0 = s_lo; s0 < s_hi; s0 += kStepChunk) {
        const int ns = min(kStepChunk, s_hi - s0);
        __syncthreads();                     // the previous chunk's entries are consumed
        if (tid < ns) {
            const int s = s0 + tid;
            bool d2, d1;
            step_due(s, c, d2, d1);
            s_set[tid] = (unsigned char)((d2 ? 1 : 0) | (d1 ? 2 : 0));
            s_base[tid] = offset_of(s, c, total);
            if (tile == 0) offsets[s + 1] = (int32_t)offset_of(s + 1, c, total);
        }
        __syncthreads();
        for (int k = 0; k < ns; ++k) {
            const int set = s_set[k];
            const bool mine = set == 0 ? in[0] : set == 1 ? in[1] : set == 2 ? in[2] : in[3];
            const int p = set == 0 ? pos[0] : set == 1 ? pos[1] : set == 2 ? pos[2] : pos[3];
            if (mine) idx[s_base[k] + p] = t;
        }
    }
}

Geo make_geo(const jano_geom& g) {
    Geo o;
    o.pf = g.pf; o.ph = g.ph; o.pw = g.pw;
    o.TF = g.F / g.pf; o.TH = g.H / g.ph; o.TW = g.W / g.pw;
    o.bf = g.bf; o.bh = g.bh; o.bw = g.bw;
    o.nBh = (g.H + g.bh - 1) / g.bh;
    o.nBw = (g.W + g.bw - 1) / g.bw;
    o.n_blocks = ((g.F + g.bf - 1) / g.bf) * o.nBh * o.nBw;
    return o;
}

}  // namespace

size_t schedule_workspace_bytes(const jano_geom& g) {
    const long long nt = (long long)(g.F / g.pf) * (g.H / g.ph) * (g.W / g.pw);
    const long long tiles = (nt + kTile - 1) / kTile;
    return align16((size_t)nt) + align16(sizeof(int) * 3 * (size_t)tiles);
}

cudaError_t launch_build_schedule(const uint8_t* block_levels, const jano_geom& g,
                                  const jano_sched_cfg& c, int32_t* offsets,
                                  int32_t* idx, uint8_t* token_levels, void* ws_base,
                                  int* err, cudaStream_t st) {
    const Geo geo = make_geo(g);
    const int n_tokens = geo.TF * geo.TH * geo.TW;
    const int n_tiles = (n_tokens + kTile - 1) / kTile;
    const Ws ws = carve(ws_base, n_tokens, n_tiles);
    count_kernel<<<n_tiles, kTile, 0, st>>>(block_levels, geo, n_tokens, token_levels, ws,
                                             n_tiles, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // step chunks: enough (tile, chunk) CTAs for two per SM, at most one chunk per step
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int chunks = std::max(1, std::min(c.T, (2 * sms + n_tiles - 1) / n_tiles));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)n_tiles, (unsigned)chunks, 1);
    cfg.blockDim = dim3(kTile, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, write_kernel, ws, n_tokens, n_tiles, c, offsets, idx);
}

}  // namespace jano
