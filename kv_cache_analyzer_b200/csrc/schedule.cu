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
//   2. scan    one CTA: per-level exclusive prefixes over tiles, per-step
//              totals and the offsets[] prefix over steps;
//   3. write   one CTA per (tile, 8 steps): the tile's tokens ranked once in
//              each of the four possible due sets (ballot + popc + one warp
//              scan per set), then ascending stores of the due ids per step.
// Scratch (caller-provided): token levels [n_tokens] u8, counts/prefixes
// [3][n_tiles] int32 each.
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
    int* pre;                     // [3][n_tiles]
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

Ws carve(void* base, long long n_tokens, int n_tiles) {
    char* p = static_cast<char*>(base);
    Ws w;
    w.tok = reinterpret_cast<uint8_t*>(p);
    p += align16((size_t)n_tokens);
    w.cnt = reinterpret_cast<int*>(p);
    p += align16(sizeof(int) * 3 * (size_t)n_tiles);
    w.pre = reinterpret_cast<int*>(p);
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

__global__ void __launch_bounds__(kTile)
scan_kernel(Ws ws, int n_tiles, jano_sched_cfg c, int32_t* __restrict__ offsets) {
    __shared__ int wsum[32];
    __shared__ int s_tot[3];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // per level: exclusive prefix of the tile counts, chunk by chunk
    for (int l = 0; l < 3; ++l) {
        int run = 0;
        for (int base = 0; base < n_tiles; base += kTile) {
            const int i = base + tid;
            const int v = i < n_tiles ? ws.cnt[l * n_tiles + i] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            if (lane == 31) wsum[warp] = incl;
            __syncthreads();
            int wpre = 0, tot = 0;
            for (int w = 0; w < 32; ++w) {
                if (w < warp) wpre += wsum[w];
                tot += wsum[w];
            }
            if (i < n_tiles) ws.pre[l * n_tiles + i] = run + wpre + incl - v;
            run += tot;
            __syncthreads();
        }
        if (tid == 0) s_tot[l] = run;
        __syncthreads();
    }
    // per step counts and their prefix (T is small: a serial loop in one thread)
    if (tid == 0) {
        long long acc = 0;
        offsets[0] = 0;
        for (int s = 0; s < c.T; ++s) {
            bool d2, d1;
            step_due(s, c, d2, d1);
            acc += s_tot[2] + (d2 ? s_tot[1] : 0) + (d1 ? s_tot[0] : 0);
            offsets[s + 1] = (int32_t)acc;
        }
    }
}

// The due set of a step is one of four unions of levels: {3}, {3,2}, {3,1},
// {3,2,1} (set id = due2 | due1 << 1).  Each CTA ranks its tile's tokens in
// all four once (ballots + one warp scan per set) and then writes the lists
// of kStepsPerCta consecutive steps from those ranks.
constexpr int kStepsPerCta = 8;

__global__ void __launch_bounds__(kTile)
write_kernel(Ws ws, int n_tokens, int n_tiles, jano_sched_cfg c,
             const int32_t* __restrict__ offsets, int32_t* __restrict__ idx) {
    __shared__ int wc[4][32];
    __shared__ int wpre[4][32];
    __shared__ int tpre[3];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tile = blockIdx.x;
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
    if (tid < 3) tpre[tid] = ws.pre[tid * n_tiles + tile];
    __syncthreads();
    if (warp < 4) {
        const int v = wc[warp][lane];
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += y;
        }
        wpre[warp][lane] = incl - v;
    }
    __syncthreads();
    const int s_end = min(c.T, (int)(blockIdx.y + 1) * kStepsPerCta);
    for (int s = blockIdx.y * kStepsPerCta; s < s_end; ++s) {
        bool d2, d1;
        step_due(s, c, d2, d1);
        const int set = (d2 ? 1 : 0) | (d1 ? 2 : 0);
        if (in[set]) {
            const long long base = (long long)offsets[s] + tpre[2] + (d2 ? tpre[1] : 0) + (d1 ? tpre[0] : 0);
            idx[base + wpre[set][warp] + rank[set]] = t;
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
    return align16((size_t)nt) + 2 * align16(sizeof(int) * 3 * (size_t)tiles);
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
    scan_kernel<<<1, kTile, 0, st>>>(ws, n_tiles, c, offsets);
    write_kernel<<<dim3(n_tiles, (c.T + kStepsPerCta - 1) / kStepsPerCta), kTile, 0, st>>>(
        ws, n_tokens, n_tiles, c, offsets, idx);
    return cudaGetLastError();
}

}  // namespace jano
