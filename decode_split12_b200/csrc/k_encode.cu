// k_encode.cu -- Split12 encoder kernels.
//
// Trained weights reuse a narrow set of exponents, so each 128-weight tile
// gets a base whose 15-exponent window holds as many of its weights as
// possible; those weights keep a 4-bit code, the rest become exact escapes
// ("Lossless LLM Weight Compression vs 8-bit GGUF", "What did the GLM-5.2
// experiment actually prove?": short fixed codes for common symbols, rare
// ones to an exact escape stream; "GPU 友善 12 位無損 BF16 壓縮格式",
// technical deep dive: 128-weight blocks sharing a base).
//
// W is read once in full.  The raw, code and base planes sit at offsets that
// do not depend on the escape count, so they are written in that one pass;
// only the escape stream and its offsets need the escape counts of all
// earlier tiles.
//   E1 (tile_kernel): 32 consecutive tiles per group, two at a time (a
//       half-warp per tile, one 16-byte load per lane, the next pair's load
//       in flight).  A tile whose exponents span at most 15 values fits one
//       window whole, and its base is the smallest b whose window reaches
//       the largest exponent; otherwise (the tile has escapes) the window is
//       searched over the exponent histogram for the b in [0, 241] that holds
//       the most weights, ties to the smallest b.  Writes the raw bytes,
//       code nibbles, base, the tile's escape count and the warp's total.
//       The warps of a grid of a few blocks per SM take the groups in turn.
//   E3 (escape_kernel): each block first sums the escape counts of all
//       groups before its own (integer, deterministic; no separate scan
//       pass), block 0 also the grand total n_esc.  Then per warp, the
//       escape offsets of its 32 tiles (a warp scan of their counts from
//       the group's offset), then the
//       escape values of the few tiles that have any, read from W again, in
//       row-major order; the first block also writes the header and the zero
//       padding.
//   The host then reads n_esc once (one stream synchronisation) and checks
//   the capacity: escapes past the end of the destination are not written,
//   and the call reports the size it needs.
#include <algorithm>

#include "s12_device.cuh"
#include "s12_launch.h"

namespace s12 {

constexpr int kEncWarps = 8;
constexpr int kTilesPerWarp = 32;

__device__ __forceinline__ uint32_t exp_field(uint32_t w16) { return (w16 >> 7) & 0xFFu; }

struct EncodeParams {
    const uint16_t *__restrict__ w;
    uint64_t n_tiles;
    uint8_t *base_out;      // nullable (size query)
    uint32_t *warp_cnt;     // [n_groups]: E1 writes totals, E2 turns them into offsets
    unsigned long long *total;
    uint8_t *tile_cnt;      // [n_tiles]: escapes of each tile (E1 -> E3)
    uint64_t n_groups;
    // pack outputs
    uint8_t *raw;
    uint8_t *code;
    uint32_t *esc_off;
    uint16_t *esc;
    // E3's block 0 also writes the header and the zero padding
    uint8_t *dst;
    uint64_t rows, cols, dst_cap;
};

// A warp works on two tiles at a time: lanes 0-15 hold tile t (8 weights
// each, one 16-byte load), lanes 16-31 tile t+1.  `valid`: the half-warp's
// tile exists.
__device__ __forceinline__ uint4 load_pair(const EncodeParams &p, uint64_t t0, int lane, uint64_t t_end) {
    const uint64_t t = t0 + static_cast<uint64_t>(lane >> 4);
    if (t >= t_end) return make_uint4(0, 0, 0, 0);
    return __ldcs(reinterpret_cast<const uint4 *>(p.w + t * kTile) + (lane & 15));
}

__device__ __forceinline__ uint32_t weight_k(const uint4 &v, int k) {
    const uint32_t w = k < 2 ? v.x : k < 4 ? v.y : k < 6 ? v.z : v.w;
    return (k & 1) ? w >> 16 : w & 0xFFFFu;
}

// Four weights (two 32-bit words, two weights each) as byte lanes: lo4 holds
// their low bytes, hi4 their high bytes (weight k in byte k).
__device__ __forceinline__ void split4(uint32_t x, uint32_t y, uint32_t &lo4, uint32_t &hi4) {
    lo4 = prmt(x, y, 0x6420u);
    hi4 = prmt(x, y, 0x7531u);
}

// The exponent fields of those four weights, one per byte.
__device__ __forceinline__ uint32_t exps4(uint32_t lo4, uint32_t hi4) {
    return ((hi4 << 1) & 0xFEFEFEFEu) | ((lo4 >> 7) & 0x01010101u);
}

// Base of the half-warp's tile: the b in [0, 241] whose window [b, b+14]
// holds the most exponents, ties to the smallest b.  hist: the half-warp's
// 256 counters, pref: its 272-word prefix array (shared memory).  Every lane
// of the warp calls it.
// (kept out of line: it is the rare path, taken by tiles with escapes)
__device__ __noinline__ uint32_t tile_base(uint4 v, bool valid, uint32_t *hist, uint32_t *pref, int lane,
                                           uint32_t *in_window) {
    const int hl = lane & 15, half = lane >> 4;
    const unsigned hmask = 0xFFFFu << (16 * half);
    // this lane's 16 counters to zero
    uint4 *h4 = reinterpret_cast<uint4 *>(hist + 16 * hl);
#pragma unroll
    for (int k = 0; k < 4; ++k) h4[k] = make_uint4(0, 0, 0, 0);
    __syncwarp();
    if (valid) {
#pragma unroll
        for (int k = 0; k < 8; ++k) atomicAdd(&hist[exp_field(weight_k(v, k))], 1u);
    }
    __syncwarp();
    // exclusive prefix: P[k] = weights with exponent < 16*hl + k
    uint32_t P[16];
    uint32_t run = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 c = h4[q];
        P[4 * q] = run;
        run += c.x;
        P[4 * q + 1] = run;
        run += c.y;
        P[4 * q + 2] = run;
        run += c.z;
        P[4 * q + 3] = run;
        run += c.w;
    }
    uint32_t incl = run;
#pragma unroll
    for (int d = 1; d < 16; d <<= 1) {
        const uint32_t t = __shfl_up_sync(0xFFFFFFFFu, incl, d, 16);
        if (hl >= d) incl += t;
    }
    const uint32_t lane_base = incl - run;
    uint4 *p4 = reinterpret_cast<uint4 *>(pref + 16 * hl);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        p4[q] = make_uint4(lane_base + P[4 * q], lane_base + P[4 * q + 1], lane_base + P[4 * q + 2],
                           lane_base + P[4 * q + 3]);
    if (hl == 15) pref[256] = incl;
    __syncwarp();
    // window counts pref[b + 15] - pref[b] for b = 16*hl + k: index b + 15 is
    // this lane's last entry for k = 0 and the next lane's entry k - 1 after
    uint32_t N[16];
    const uint4 *n4 = reinterpret_cast<const uint4 *>(pref + 16 * hl + 16);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 c = n4[q];
        N[4 * q] = c.x;
        N[4 * q + 1] = c.y;
        N[4 * q + 2] = c.z;
        N[4 * q + 3] = c.w;
    }
    uint32_t best = 0;  // key = count << 8 | (255 - b): max -> most weights, then smallest b
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int b = 16 * hl + k;
        if (b <= kMaxBase) {
            const uint32_t top = k == 0 ? lane_base + P[15] : N[k - 1];
            const uint32_t c = top - (lane_base + P[k]);
            const uint32_t key = (c << 8) | static_cast<uint32_t>(255 - b);
            best = key > best ? key : best;
        }
    }
    best = __reduce_max_sync(hmask, best);
    __syncwarp();
    *in_window = best >> 8;
    return 255u - (best & 0xFFu);
}

// E1 for one group of kTilesPerWarp tiles (one warp).
__device__ __forceinline__ void encode_group(const EncodeParams &p, uint64_t group, uint32_t (*hist)[256],
                                             uint32_t (*pref)[272], int lane, int half, int hl) {
    const uint64_t t_begin = group * kTilesPerWarp;
    const uint64_t t_end = min(t_begin + kTilesPerWarp, p.n_tiles);
    uint32_t sum = 0;
    auto work = [&](const uint4 &v, uint64_t t0) {
        const uint64_t t = t0 + static_cast<uint64_t>(half);
        const bool valid = t < t_end;
        // byte lanes: weights 0-3 (a) and 4-7 (b) of the lane's eight
        uint32_t la, ha, lb, hb;
        split4(v.x, v.y, la, ha);
        split4(v.z, v.w, lb, hb);
        const uint32_t ea = exps4(la, ha), eb = exps4(lb, hb);
        // the tile's smallest and largest exponent
        uint32_t mx = __vmaxu4(ea, eb), mn = __vminu4(ea, eb);
        mx = __vmaxu4(mx, prmt(mx, 0u, 0x1032u));
        mx = __vmaxu4(mx, prmt(mx, 0u, 0x2301u));
        mn = __vminu4(mn, prmt(mn, 0u, 0x1032u));
        mn = __vminu4(mn, prmt(mn, 0u, 0x2301u));
        // over the half-warp: largest exponent in the high 16 bits, 255 -
        // smallest in the low 16, reduced together by 16-bit maxima
        uint32_t key = ((mx & 0xFFu) << 16) | (255u - (mn & 0xFFu));
#pragma unroll
        for (int d = 1; d < 16; d <<= 1) key = __vmaxu2(key, __shfl_xor_sync(0xFFFFFFFFu, key, d));
        const uint32_t emax = key >> 16, emin = 255u - (key & 0xFFFFu);
        uint32_t b = emax > 14u ? emax - 14u : 0u, inw = kTile;
        if (__any_sync(0xFFFFFFFFu, valid && emax - emin > 14u))
            b = tile_base(v, valid, hist[half], pref[half], lane, &inw);
        if (valid) sum += kTile - inw;
        if (!p.raw || !valid) return;  // size query: counts only
        // raw byte = sign | mantissa
        const uint32_t raw0 = (la & 0x7F7F7F7Fu) | (ha & 0x80808080u);
        const uint32_t raw1 = (lb & 0x7F7F7F7Fu) | (hb & 0x80808080u);
        // code = exponent - base when in [0, 14], else 15 (escape)
        const uint32_t B4 = b * 0x01010101u;
        const uint32_t da = __vsub4(ea, B4), db = __vsub4(eb, B4);
        const uint32_t ina = __vcmpleu4(da, 0x0E0E0E0Eu), inb = __vcmpleu4(db, 0x0E0E0E0Eu);
        const uint32_t ca = (da & ina) | (0x0F0F0F0Fu & ~ina), cb = (db & inb) | (0x0F0F0F0Fu & ~inb);
        // nibble k = code of weight k
        const uint32_t codes = prmt(ca | (ca >> 4), cb | (cb >> 4), 0x6420u);
        reinterpret_cast<uint2 *>(p.raw + t * kTile)[hl] = make_uint2(raw0, raw1);
        reinterpret_cast<uint32_t *>(p.code + t * (kTile / 2))[hl] = codes;
        if (hl == 0) {
            p.base_out[t] = static_cast<uint8_t>(b);
            p.tile_cnt[t] = static_cast<uint8_t>(kTile - inw);
        }
    };
    uint4 a = load_pair(p, t_begin, lane, t_end);
    for (uint64_t t = t_begin; t < t_end; t += 4) {
        const uint4 b = load_pair(p, t + 2, lane, t_end);
        work(a, t);
        if (t + 2 >= t_end) break;
        a = load_pair(p, t + 4, lane, t_end);
        work(b, t + 2);
    }
    // (lane 0 counted the first tile of each pair, lane 16 the second)
    sum = hl == 0 ? sum : 0u;
    sum += __shfl_xor_sync(0xFFFFFFFFu, sum, 16);
    if (lane == 0) p.warp_cnt[group] = sum;
}

// E1: see the file comment.
__global__ void __launch_bounds__(32 * kEncWarps, 3) tile_kernel(EncodeParams p) {
    __shared__ __align__(16) uint32_t s_hist[kEncWarps][2][256];
    __shared__ __align__(16) uint32_t s_pref[kEncWarps][2][272];
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5, half = lane >> 4, hl = lane & 15;
    // warps take groups in turn (a grid of a few blocks per SM), so the
    // occasional tile that needs the window search is spread over the warps
    const uint64_t n_warps = static_cast<uint64_t>(gridDim.x) * kEncWarps;
    for (uint64_t group = static_cast<uint64_t>(blockIdx.x) * kEncWarps + wi; group < p.n_groups; group += n_warps)
        encode_group(p, group, s_hist[wi], s_pref[wi], lane, half, hl);
}

// Sum of cnt[0 .. n) by the threads of one block (any n; deterministic).
__device__ unsigned long long block_sum(const uint32_t *cnt, uint64_t n, unsigned long long *red) {
    unsigned long long s = 0;
    for (uint64_t i = threadIdx.x; i < n; i += blockDim.x) s += cnt[i];
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, d);
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
    __syncthreads();  // red may hold an earlier call's values
    if (lane == 0) red[wi] = s;
    __syncthreads();
    unsigned long long t = 0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) t += red[i];
    return t;
}

// The header (64 bytes in use, the rest of its 256 zero) and the zero padding
// after every plane, by the threads of one block; the escape count comes from
// grand total.  Padding past dst_cap is not written.
__device__ void write_header_and_padding(const EncodeParams &p, uint64_t n_esc) {
    const Geometry g = geometry(p.rows, p.cols, n_esc);
    uint32_t *h = reinterpret_cast<uint32_t *>(p.dst);
    for (int i = threadIdx.x; i < 64; i += blockDim.x) {
        uint32_t v = 0;
        switch (i) {
            case 0: v = 0x00323153u; break;  // "S12\0"
            case 1: v = 1u; break;           // version
            case 2: v = static_cast<uint32_t>(p.rows); break;
            case 3: v = static_cast<uint32_t>(p.rows >> 32); break;
            case 4: v = static_cast<uint32_t>(p.cols); break;
            case 5: v = static_cast<uint32_t>(p.cols >> 32); break;
            case 6: v = static_cast<uint32_t>(kTile); break;
            case 7: v = 0u; break;  // flags
            case 8: v = static_cast<uint32_t>(n_esc); break;
            case 9: v = static_cast<uint32_t>(n_esc >> 32); break;
            default: v = 0u;
        }
        h[i] = v;
    }
    const uint64_t gaps[5][2] = {{g.off_raw + g.rows * g.cols, g.off_code},
                                 {g.off_code + g.rows * g.cols / 2, g.off_base},
                                 {g.off_base + g.n_tiles, g.off_esc_off},
                                 {g.off_esc_off + 4 * (g.n_tiles + 1), g.off_esc},
                                 {g.off_esc + 2 * n_esc, g.total}};
    for (int k = 0; k < 5; ++k) {
        const uint64_t end = gaps[k][1] < p.dst_cap ? gaps[k][1] : p.dst_cap;
        for (uint64_t i = gaps[k][0] + threadIdx.x; i < end; i += blockDim.x) p.dst[i] = 0;
    }
}

// E3: see the file comment.  Lane i of a warp stands for tile i of the
// warp's 32.
__global__ void __launch_bounds__(32 * kEncWarps) escape_kernel(EncodeParams p) {
    __shared__ unsigned long long s_red[kEncWarps];
    __shared__ uint32_t s_off[kEncWarps];
    const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
    const uint64_t group0 = static_cast<uint64_t>(blockIdx.x) * kEncWarps;
    // escapes before this block's first group: the sum of the earlier
    // groups' counts (every block sums its own prefix: no scan pass, and
    // the result does not depend on the order blocks run in)
    const unsigned long long before = block_sum(p.warp_cnt, group0, s_red);
    if (blockIdx.x == 0) {
        // the grand total, for the header, the padding and the host
        const unsigned long long total = block_sum(p.warp_cnt, p.n_groups, s_red);
        if (threadIdx.x == 0) *p.total = total;
        if (p.dst) write_header_and_padding(p, total);
    }
    if (!p.dst) return;  // size query: the total only
    if (threadIdx.x < kEncWarps) {
        const uint64_t g = group0 + threadIdx.x;
        s_off[threadIdx.x] = g < p.n_groups ? p.warp_cnt[g] : 0u;
    }
    __syncthreads();
    const uint64_t group = group0 + wi;
    if (group >= p.n_groups) return;
    uint32_t off0 = static_cast<uint32_t>(before);
    for (int i = 0; i < wi; ++i) off0 += s_off[i];
    const Geometry g0 = geometry(p.rows, p.cols, 0);
    const uint64_t esc_cap = (p.dst_cap - g0.off_esc) / 2;
    const uint64_t t_begin = group * kTilesPerWarp;
    const uint64_t t = t_begin + static_cast<uint64_t>(lane);
    const bool valid = t < p.n_tiles;
    const uint32_t cnt = valid ? p.tile_cnt[t] : 0u;
    uint32_t incl = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, incl, d);
        if (lane >= d) incl += x;
    }
    if (valid) p.esc_off[t] = off0 + incl - cnt;
    if (t + 1 == p.n_tiles) p.esc_off[p.n_tiles] = off0 + incl;
    // the escape values, tile by tile (lane k holds weights 4k .. 4k+3)
    unsigned todo = __ballot_sync(0xFFFFFFFFu, cnt != 0);
    while (todo) {
        const int i = __ffs(todo) - 1;
        todo &= todo - 1;
        const uint64_t tt = t_begin + static_cast<uint64_t>(i);
        const uint32_t first = __shfl_sync(0xFFFFFFFFu, off0 + incl - cnt, i);
        const uint32_t b = p.base_out[tt];
        const uint2 v = __ldcs(reinterpret_cast<const uint2 *>(p.w + tt * kTile) + lane);
        const uint32_t wv[4] = {v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16};
        uint32_t m = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (exp_field(wv[k]) - b > 14u) m |= 1u << k;  // wraps when the exponent is below b
        const uint32_t n = static_cast<uint32_t>(__popc(m));
        uint32_t rank = n;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const uint32_t x = __shfl_up_sync(0xFFFFFFFFu, rank, d);
            if (lane >= d) rank += x;
        }
        uint64_t idx = static_cast<uint64_t>(first) + rank - n;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (m & (1u << k)) {
                if (idx < esc_cap) p.esc[idx] = static_cast<uint16_t>(wv[k]);
                ++idx;
            }
    }
}

size_t encode_ws_bytes(int64_t rows, int64_t cols) {
    if (rows <= 0 || cols <= 0 || cols % kTile) return 0;
    const uint64_t n_tiles = static_cast<uint64_t>(rows) * (cols / kTile);
    const uint64_t n_groups = (n_tiles + kTilesPerWarp - 1) / kTilesPerWarp;
    return static_cast<size_t>(align_up(16 + 4 * n_groups, 256) + align_up(n_tiles, 256));
}

int launch_encode(const uint16_t *w, int64_t rows, int64_t cols, void *dst, size_t dst_cap, size_t *bytes_out,
                  void *ws, size_t ws_bytes, cudaStream_t stream) {
    const uint64_t R = static_cast<uint64_t>(rows), C = static_cast<uint64_t>(cols);
    const uint64_t n_tiles = R * (C / kTile);
    const uint64_t n_groups = (n_tiles + kTilesPerWarp - 1) / kTilesPerWarp;
    if (ws_bytes < encode_ws_bytes(rows, cols)) return S12_ERR_CAPACITY;
    const Geometry g0 = geometry(R, C, 0);
    // a destination smaller than the escape-free size is not written: the
    // call then works as a size query and reports S12_ERR_CAPACITY
    const bool too_small = dst && dst_cap < g0.total;
    uint8_t *d = too_small ? nullptr : static_cast<uint8_t *>(dst);

    EncodeParams p;
    p.w = w;
    p.n_tiles = n_tiles;
    p.base_out = d ? d + g0.off_base : nullptr;
    p.total = static_cast<unsigned long long *>(ws);
    p.warp_cnt = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + 16);
    p.tile_cnt = static_cast<uint8_t *>(ws) + align_up(16 + 4 * n_groups, 256);
    p.n_groups = n_groups;
    p.raw = d ? d + g0.off_raw : nullptr;
    p.code = d ? d + g0.off_code : nullptr;
    p.esc_off = d ? reinterpret_cast<uint32_t *>(d + g0.off_esc_off) : nullptr;
    p.esc = d ? reinterpret_cast<uint16_t *>(d + g0.off_esc) : nullptr;
    p.dst = d;
    p.rows = R;
    p.cols = C;
    p.dst_cap = dst_cap;

    // E1 and E3 back to back (a size query runs only E3's total), then one
    // synchronisation to read the escape total
    const unsigned grid = static_cast<unsigned>((n_groups + kEncWarps - 1) / kEncWarps);
    int sms = 0;
    if (device_sms(&sms) != cudaSuccess) return S12_ERR_CUDA;
    const unsigned grid1 = static_cast<unsigned>(std::min<uint64_t>(grid, static_cast<uint64_t>(3 * sms)));
    tile_kernel<<<grid1, 32 * kEncWarps, 0, stream>>>(p);
    escape_kernel<<<d ? grid : 1u, 32 * kEncWarps, 0, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return S12_ERR_CUDA;
    unsigned long long n_esc = 0;
    if (cudaMemcpyAsync(&n_esc, p.total, sizeof n_esc, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return S12_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return S12_ERR_CUDA;
    const Geometry g = geometry(R, C, n_esc);
    *bytes_out = static_cast<size_t>(g.total);
    if (too_small || (d && dst_cap < g.total)) return S12_ERR_CAPACITY;
    return S12_OK;
}

}  // namespace s12
