// Plan kernels: coordinate-block partition and coordinate hash + window neighbour lists.
//
// Direct3D-S2 model page, "What is Direct3D-S2?": SSA partitions sparse tokens by their 3D
// coordinates. Direct3D-S2 summary page, "Technical principles", SSA item: compression per
// block, block selection, local window.
//
// Partition: every token gets a dense block key (sequence base + (bx*GBy + by)*GBz + bz); a
// histogram over the dense key space, an occupancy scan and a block-size scan give the block
// CSR with blocks in lexicographic (bx, by, bz) order; a counting scatter followed by a per-block
// sort puts the tokens of each block in ascending index order. Window: tokens are inserted in
// an open-addressing hash of packed (sequence, x, y, z); each token probes the (2r+1)^3 cells
// around it (count pass, scan, fill pass with a per-row sort).
#include <algorithm>

#include "common.cuh"

namespace ssa {

namespace {

constexpr int kThreads = 256;

inline unsigned grid_for(int64_t n, int threads = kThreads) {
    int64_t g = cdiv(n > 0 ? n : 1, threads);
    return (unsigned)std::min<int64_t>(g, 1 << 30);
}

// Sorts buf[0..cap) ascending with one warp (cap a power of two).
__device__ void warp_bitonic_sort(int32_t* buf, int cap) {
    const int lane = threadIdx.x & 31;
    for (int k = 2; k <= cap; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = lane; i < cap; i += 32) {
                int ixj = i ^ j;
                if (ixj > i) {
                    int32_t a = buf[i], b = buf[ixj];
                    bool up = (i & k) == 0;
                    if ((a > b) == up) {
                        buf[i] = b;
                        buf[ixj] = a;
                    }
                }
            }
            __syncwarp();
        }
    }
}

__device__ __forceinline__ int32_t hash_find(const uint64_t* __restrict__ hkeys,
                                             const int32_t* __restrict__ hvals, uint64_t hmask,
                                             uint64_t key) {
    uint64_t slot = mix64(key) & hmask;
    for (uint64_t probe = 0; probe <= hmask; ++probe) {
        uint64_t k = hkeys[slot];
        if (k == key) return hvals[slot];
        if (k == kEmptyCell) return -1;
        slot = (slot + 1) & hmask;
    }
    return -1;
}

// Validates coordinates, computes dense block keys, counts tokens per key and inserts every token
// in the coordinate hash (duplicates flagged).
__global__ void k_keys_and_hash(const int32_t* __restrict__ coords, int64_t N,
                                const SeqInfo* __restrict__ seqs, int B,
                                int32_t* __restrict__ tok_key, int32_t* __restrict__ key_cnt,
                                uint64_t* __restrict__ hkeys, int32_t* __restrict__ hvals,
                                uint64_t hmask, int32_t* __restrict__ status) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N) return;
    int s = find_seq(seqs, B, i);
    const SeqInfo q = seqs[s];
    int32_t x = coords[3 * i], y = coords[3 * i + 1], z = coords[3 * i + 2];
    if (x < 0 || y < 0 || z < 0 || x >= q.gx || y >= q.gy || z >= q.gz) {
        atomicOr(status, DEV_COORD_RANGE);
        tok_key[i] = -1;
        return;
    }
    int64_t key = q.dense_base + ((int64_t)(x / kBlockEdge) * q.gby + (y / kBlockEdge)) * q.gbz +
                  (z / kBlockEdge);
    tok_key[i] = (int32_t)key;
    atomicAdd(&key_cnt[key], 1);
    uint64_t cell = pack_cell(s, x, y, z);
    uint64_t slot = mix64(cell) & hmask;
    for (uint64_t probe = 0; probe <= hmask; ++probe) {
        unsigned long long prev = atomicCAS((unsigned long long*)&hkeys[slot],
                                            (unsigned long long)kEmptyCell,
                                            (unsigned long long)cell);
        if (prev == kEmptyCell) {
            hvals[slot] = (int32_t)i;
            return;
        }
        if (prev == cell) {
            atomicOr(status, DEV_DUPLICATE);
            return;
        }
        slot = (slot + 1) & hmask;
    }
    atomicOr(status, DEV_TOO_LARGE);  // table full: cannot happen with 2N slots
}

__global__ void k_occupied(const int32_t* __restrict__ key_cnt, int64_t G, int32_t* __restrict__ flag) {
    int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k < G) flag[k] = key_cnt[k] > 0;
}

// For every occupied dense key: its block index, size, padded size, coordinates and sequence.
__global__ void k_blocks(const int32_t* __restrict__ key_cnt, const int32_t* __restrict__ bidx,
                         int64_t G, const SeqInfo* __restrict__ seqs, int B,
                         int32_t* __restrict__ key2blk, int32_t* __restrict__ blk_cnt,
                         int32_t* __restrict__ blk_pcnt, int32_t* __restrict__ blk_coord,
                         int32_t* __restrict__ blk_seq) {
    int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= G) return;
    int32_t c = key_cnt[k];
    if (c == 0) {
        key2blk[k] = -1;
        return;
    }
    int32_t b = bidx[k];
    key2blk[k] = b;
    blk_cnt[b] = c;
    blk_pcnt[b] = (int32_t)round_up(c, kPad);
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (seqs[mid].dense_base <= k) lo = mid; else hi = mid - 1;
    }
    const SeqInfo q = seqs[lo];
    int64_t local = k - q.dense_base;
    blk_coord[3 * b + 2] = (int32_t)(local % q.gbz);
    blk_coord[3 * b + 1] = (int32_t)((local / q.gbz) % q.gby);
    blk_coord[3 * b + 0] = (int32_t)(local / ((int64_t)q.gbz * q.gby));
    blk_seq[b] = lo;
}

// One warp per token: probe every cell of the (2r+1)^3 cube, count (fill == false) or write the
// found neighbours sorted ascending (fill == true).
template <bool kFill>
__global__ void k_neighbours(const int32_t* __restrict__ coords, int64_t N,
                             const SeqInfo* __restrict__ seqs, int B, int r,
                             const uint64_t* __restrict__ hkeys, const int32_t* __restrict__ hvals,
                             uint64_t hmask, int32_t* __restrict__ nbr_cnt,
                             const int32_t* __restrict__ nbr_off, int32_t* __restrict__ nbr_idx,
                             int cap, int32_t* __restrict__ status) {
    extern __shared__ int32_t sbuf[];
    const int lane = threadIdx.x & 31;
    const int wib = threadIdx.x >> 5;
    int64_t i = (int64_t)blockIdx.x * (blockDim.x >> 5) + wib;
    if (i >= N) return;
    int32_t* buf = sbuf + (int64_t)wib * cap;
    int s = find_seq(seqs, B, i);
    const SeqInfo q = seqs[s];
    int32_t x = coords[3 * i], y = coords[3 * i + 1], z = coords[3 * i + 2];
    const int w = 2 * r + 1;
    const int cube = w * w * w;
    int count = 0;
    for (int o0 = 0; o0 < cube; o0 += 32) {
        int o = o0 + lane;
        int32_t j = -1;
        if (o < cube) {
            int dz = o % w - r, dy = (o / w) % w - r, dx = o / (w * w) - r;
            int32_t xx = x + dx, yy = y + dy, zz = z + dz;
            if (xx >= 0 && yy >= 0 && zz >= 0 && xx < q.gx && yy < q.gy && zz < q.gz)
                j = hash_find(hkeys, hvals, hmask, pack_cell(s, xx, yy, zz));
        }
        unsigned found = __ballot_sync(0xffffffffu, j >= 0);
        if (kFill && j >= 0) buf[count + __popc(found & ((1u << lane) - 1))] = j;
        count += __popc(found);
    }
    if (!kFill) {
        if (lane == 0) nbr_cnt[i] = count;
        return;
    }
    __syncwarp();
    if (count != nbr_off[i + 1] - nbr_off[i]) {
        if (lane == 0) atomicOr(status, DEV_BAD_INDEX);
        return;
    }
    for (int t = count + lane; t < cap; t += 32) buf[t] = 0x7fffffff;
    __syncwarp();
    warp_bitonic_sort(buf, cap);
    for (int t = lane; t < count; t += 32) nbr_idx[nbr_off[i] + t] = buf[t];
}

// Counting scatter of tokens into their blocks (order inside a block fixed by k_sort_blocks).
__global__ void k_scatter(const int32_t* __restrict__ tok_key, const int32_t* __restrict__ key2blk,
                          int64_t N, const int32_t* __restrict__ blk_off,
                          int32_t* __restrict__ blk_fill, int32_t* __restrict__ perm,
                          int32_t* __restrict__ tok_blk) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N) return;
    int32_t b = key2blk[tok_key[i]];
    tok_blk[i] = b;
    int32_t pos = blk_off[b] + atomicAdd(&blk_fill[b], 1);
    perm[pos] = (int32_t)i;
}

// One warp per block: sort the block's slice of perm ascending (a block holds at most 512 cells).
__global__ void k_sort_blocks(int32_t* __restrict__ perm, const int32_t* __restrict__ blk_off,
                              int64_t Mb) {
    __shared__ int32_t sbuf[8][512];
    const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
    int64_t b = (int64_t)blockIdx.x * 8 + wib;
    if (b >= Mb) return;
    int32_t lo = blk_off[b], n = blk_off[b + 1] - lo;
    int cap = 32;
    while (cap < n) cap <<= 1;
    int32_t* buf = sbuf[wib];
    for (int t = lane; t < cap; t += 32) buf[t] = t < n ? perm[lo + t] : 0x7fffffff;
    __syncwarp();
    warp_bitonic_sort(buf, cap);
    for (int t = lane; t < n; t += 32) perm[lo + t] = buf[t];
}

// Sorted and padded positions of every token, and the per-row tables of the padded layout.
__global__ void k_positions(const int32_t* __restrict__ perm, const int32_t* __restrict__ tok_blk,
                            const int32_t* __restrict__ blk_off, const int32_t* __restrict__ blk_poff,
                            const int32_t* __restrict__ coords, int64_t N,
                            int32_t* __restrict__ tok_pos, int32_t* __restrict__ spos_tok,
                            int4* __restrict__ scoord) {
    int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (p >= N) return;
    int32_t i = perm[p];
    int32_t b = tok_blk[i];
    int32_t sp = blk_poff[b] + ((int32_t)p - blk_off[b]);
    tok_pos[i] = (int32_t)p;
    spos_tok[sp] = i;
    scoord[sp] = make_int4(coords[3 * i], coords[3 * i + 1], coords[3 * i + 2], b);
}

// (first 8-row group, tokens) of every block, for the attention kernel's union of selected blocks
__global__ void k_block_info(const int32_t* __restrict__ blk_off, const int32_t* __restrict__ blk_poff,
                             int64_t Mb, int2* __restrict__ info) {
    const int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (b < Mb) info[b] = make_int2(blk_poff[b] >> 3, blk_off[b + 1] - blk_off[b]);
}

// One CTA per sequence. The sequence's blocks of at most kPoolMaxTokens tokens get consecutive
// rows of its pool in block order: tpool[b] = first row relative to the pool, -1 for the other
// blocks; ptok[s] = rows of the pool (its tokens).
__global__ void __launch_bounds__(256) k_tiny_pool(const int32_t* __restrict__ blk_off,
                                                   const int32_t* __restrict__ seq_blk,
                                                   int32_t* __restrict__ tpool, int32_t* __restrict__ ptok) {
    __shared__ int wsum[8];
    __shared__ int carry;
    const int s = blockIdx.x, t = threadIdx.x, lane = t & 31, w = t >> 5;
    const int32_t b0 = seq_blk[s], b1 = seq_blk[s + 1];
    if (t == 0) carry = 0;
    __syncthreads();
    for (int32_t base = b0; base < b1; base += 256) {
        const int32_t b = base + t;
        const int32_t n = b < b1 ? blk_off[b + 1] - blk_off[b] : 0;
        const int v = (b < b1 && n <= kPoolMaxTokens) ? n : 0;
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[w] = x;
        __syncthreads();
        int before = carry, total = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            before += i < w ? wsum[i] : 0;
            total += wsum[i];
        }
        if (b < b1) tpool[b] = n <= kPoolMaxTokens ? before + x - v : -1;
        __syncthreads();
        if (t == 0) carry += total;
        __syncthreads();
    }
    if (t == 0) ptok[s] = carry;
}

__global__ void k_fill_i32(int32_t* __restrict__ a, int64_t n, int32_t v) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) a[i] = v;
}

__global__ void k_fill_int4(int4* __restrict__ a, int64_t n, int4 v) {
    int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) a[i] = v;
}

// Per query tile (<= 128 consecutive sorted tokens of one sequence): the union of the window
// neighbourhoods of its tokens, as ascending padded rows. Candidates are the tokens of the blocks
// in the 3x3x3 block neighbourhood of every block the tile touches (r <= 8 keeps every window
// inside it); a candidate is kept if it lies within Chebyshev distance r of some tile token.
// kFill == false writes counts, and the first spill_cap rows of every tile to spill[tile];
// kFill == true writes the rows at wt_off for the tiles that held more than spill_cap rows (the
// others are copied from spill by k_copy_union).
template <bool kFill>
__global__ void k_window_union(const int32_t* __restrict__ qt_pos, const int32_t* __restrict__ qt_len,
                               const int32_t* __restrict__ qt_seq, const int32_t* __restrict__ perm,
                               const int32_t* __restrict__ tok_blk, const int32_t* __restrict__ coords,
                               const int32_t* __restrict__ blk_coord, const int32_t* __restrict__ blk_poff,
                               const int32_t* __restrict__ blk_off,
                               const int32_t* __restrict__ key2blk, const SeqInfo* __restrict__ seqs,
                               const int4* __restrict__ scoord, int r,
                               int32_t* __restrict__ wt_cnt, const int32_t* __restrict__ wt_off,
                               int32_t* __restrict__ wt_keys, int32_t* __restrict__ spill, int spill_cap) {
    if (kFill && wt_off[blockIdx.x + 1] - wt_off[blockIdx.x] <= spill_cap) return;   // copied instead
    constexpr int kCandCap = 4096;     // 27 neighbours x up to 128 distinct tile blocks, padded
    __shared__ int4 qc[kQTile];
    __shared__ int32_t cand[kCandCap];
    __shared__ int32_t tile_blocks[kQTile];
    __shared__ int32_t qblk[kQTile];
    __shared__ int32_t ncand_s, ntb_s;
    const int t = blockIdx.x;
    const int32_t p0 = qt_pos[t], len = qt_len[t];
    const SeqInfo q = seqs[qt_seq[t]];
    if (threadIdx.x == 0) { ncand_s = 0; ntb_s = 0; }
    __syncthreads();
    __shared__ int box[6];   // bounding box of the tile's tokens: min x, y, z, max x, y, z
    if (threadIdx.x < 6) box[threadIdx.x] = threadIdx.x < 3 ? 0x7fffffff : -0x7fffffff;
    __syncthreads();
    for (int a = threadIdx.x; a < len; a += blockDim.x) {
        int32_t i = perm[p0 + a];
        qc[a] = make_int4(coords[3 * i], coords[3 * i + 1], coords[3 * i + 2], 0);
        qblk[a] = tok_blk[i];
        atomicMin(&box[0], qc[a].x);
        atomicMin(&box[1], qc[a].y);
        atomicMin(&box[2], qc[a].z);
        atomicMax(&box[3], qc[a].x);
        atomicMax(&box[4], qc[a].y);
        atomicMax(&box[5], qc[a].z);
    }
    __syncthreads();
    // distinct blocks of the tile (the tile is a run of consecutive sorted tokens)
    if (threadIdx.x == 0) {
        int32_t prev = -1;
        for (int a = 0; a < len; ++a) {
            const int32_t b = qblk[a];
            if (b != prev) tile_blocks[ntb_s++] = b;
            prev = b;
        }
    }
    __syncthreads();
    // candidate blocks: 27-neighbourhoods of the tile blocks
    for (int e = threadIdx.x; e < ntb_s * 27; e += blockDim.x) {
        int32_t tb = tile_blocks[e / 27];
        int o = e % 27;
        int bx = blk_coord[3 * tb] + o / 9 - 1, by = blk_coord[3 * tb + 1] + (o / 3) % 3 - 1,
            bz = blk_coord[3 * tb + 2] + o % 3 - 1;
        if (bx < 0 || by < 0 || bz < 0 || bx >= q.gbx || by >= q.gby || bz >= q.gbz) continue;
        int32_t nb = key2blk[q.dense_base + ((int64_t)bx * q.gby + by) * q.gbz + bz];
        if (nb < 0) continue;
        cand[atomicAdd(&ncand_s, 1)] = nb;
    }
    __syncthreads();
    // sort (bitonic over the CTA) and deduplicate the candidates
    {
        const int n = ncand_s;
        int capn = 1;
        while (capn < n) capn <<= 1;
        for (int a = n + threadIdx.x; a < capn; a += blockDim.x) cand[a] = 0x7fffffff;
        __syncthreads();
        for (int k = 2; k <= capn; k <<= 1)
            for (int j = k >> 1; j > 0; j >>= 1) {
                for (int i = threadIdx.x; i < capn; i += blockDim.x) {
                    int ixj = i ^ j;
                    if (ixj > i) {
                        int32_t a = cand[i], b = cand[ixj];
                        if ((a > b) == ((i & k) == 0)) { cand[i] = b; cand[ixj] = a; }
                    }
                }
                __syncthreads();
            }
        if (threadIdx.x == 0) {
            int m = 0;
            for (int a = 0; a < n; ++a)
                if (m == 0 || cand[m - 1] != cand[a]) cand[m++] = cand[a];
            ncand_s = m;
        }
        __syncthreads();
    }
    const int ncand = ncand_s;
    // Exact window test through occupancy bitmaps: for each of the tile's blocks (up to 4), the
    // cells of its queries in a 32^3 box with origin 8 * block - r, dilated by r along z, y and x
    // (the Chebyshev ball is a box, so the dilation separates by axis). A key is in the union iff
    // its cell is set in some block's bitmap. Tiles over more blocks test every query.
    constexpr int kMaxBitmaps = 4;
    __shared__ uint32_t bmp[kMaxBitmaps][32 * 32];   // words (x, y), bit z
    __shared__ uint32_t btmp[32 * 32];
    __shared__ int4 borg[kMaxBitmaps];
    const int ntb = ntb_s;
    const bool use_bmp = ntb <= kMaxBitmaps;
    if (use_bmp) {
        for (int i = threadIdx.x; i < ntb * 1024; i += blockDim.x) (&bmp[0][0])[i] = 0u;
        if (threadIdx.x < ntb) {
            const int32_t b = tile_blocks[threadIdx.x];
            borg[threadIdx.x] = make_int4(8 * blk_coord[3 * b] - r, 8 * blk_coord[3 * b + 1] - r,
                                          8 * blk_coord[3 * b + 2] - r, 0);
        }
        __syncthreads();
        for (int a = threadIdx.x; a < len; a += blockDim.x) {
            const int32_t b = qblk[a];
            int u = 0;
            while (u < ntb - 1 && tile_blocks[u] != b) ++u;
            const int4 o = borg[u];
            atomicOr(&bmp[u][(qc[a].x - o.x) * 32 + (qc[a].y - o.y)], 1u << (qc[a].z - o.z));
        }
        __syncthreads();
        for (int u = 0; u < ntb; ++u) {
            uint32_t* B = bmp[u];
            for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
                const uint32_t w = B[i];
                uint32_t d = w;
                for (int k = 1; k <= r; ++k) d |= (w << k) | (w >> k);
                B[i] = d;
            }
            __syncthreads();
            for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
                const int x = i >> 5, y = i & 31;
                uint32_t d = 0u;
                for (int k = -r; k <= r; ++k)
                    if (y + k >= 0 && y + k < 32) d |= B[x * 32 + y + k];
                btmp[i] = d;
            }
            __syncthreads();
            for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
                const int x = i >> 5, y = i & 31;
                uint32_t d = 0u;
                for (int k = -r; k <= r; ++k)
                    if (x + k >= 0 && x + k < 32) d |= btmp[(x + k) * 32 + y];
                B[i] = d;
            }
            __syncthreads();
        }
    }
    int32_t out_base = kFill ? wt_off[t] : 0;
    const int bx0 = box[0] - r, by0 = box[1] - r, bz0 = box[2] - r;
    const int bx1 = box[3] + r, by1 = box[4] + r, bz1 = box[5] + r;
    // keys of the candidate blocks that reach the tile's box grown by r, flattened in ascending
    // block order: kb_first[cb] = first flattened key of candidate cb (0 keys if it misses). Held in
    // the dilation scratch when the bitmaps are used (at most 4 x 27 candidates), otherwise in the
    // unused bitmap area (at most 128 x 27 = 3,456 candidates).
    int32_t* kb_first = use_bmp ? reinterpret_cast<int32_t*>(btmp) : reinterpret_cast<int32_t*>(&bmp[0][0]);
    __shared__ int wsum[32];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int cb = threadIdx.x; cb < ncand; cb += blockDim.x) {
        const int32_t b = cand[cb];
        const int cx = 8 * blk_coord[3 * b], cy = 8 * blk_coord[3 * b + 1], cz = 8 * blk_coord[3 * b + 2];
        const bool miss = cx > bx1 || cx + 7 < bx0 || cy > by1 || cy + 7 < by0 || cz > bz1 || cz + 7 < bz0;
        kb_first[cb] = miss ? 0 : blk_off[b + 1] - blk_off[b];
    }
    __syncthreads();
    {
        // exclusive prefix over the candidates: a contiguous chunk per thread, then across threads
        const int cw = (ncand + blockDim.x - 1) / blockDim.x;
        const int c0 = min((int)threadIdx.x * cw, ncand), c1 = min(c0 + cw, ncand);
        int sum = 0;
        for (int cb = c0; cb < c1; ++cb) sum += kb_first[cb];
        int x = sum;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) wsum[wid] = x;
        __syncthreads();
        int off = x - sum, tot = 0;
        for (int u = 0; u < nwarps; ++u) {
            off += u < wid ? wsum[u] : 0;
            tot += wsum[u];
        }
        for (int cb = c0; cb < c1; ++cb) {
            const int n = kb_first[cb];
            kb_first[cb] = off;
            off += n;
        }
        __syncthreads();
        if (threadIdx.x == 0) kb_first[ncand] = tot;
        __syncthreads();
    }
    const int nkeys = kb_first[ncand];
    int total = 0;
    for (int c0 = 0; c0 < nkeys; c0 += blockDim.x) {
        const int k = c0 + threadIdx.x;
        bool keep = false;
        int32_t row = 0;
        if (k < nkeys) {
            int lo = 0, hi = ncand - 1;   // last candidate whose first key is <= k
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (kb_first[mid] <= k) lo = mid; else hi = mid - 1;
            }
            row = blk_poff[cand[lo]] + (k - kb_first[lo]);
            const int4 kc = scoord[row];
            if (kc.x >= bx0 && kc.x <= bx1 && kc.y >= by0 && kc.y <= by1 && kc.z >= bz0 && kc.z <= bz1) {
                if (use_bmp) {
                    for (int u = 0; u < ntb && !keep; ++u) {
                        const int4 o = borg[u];
                        const int rx = kc.x - o.x, ry = kc.y - o.y, rz = kc.z - o.z;
                        if ((unsigned)rx < 32u && (unsigned)ry < 32u && (unsigned)rz < 32u)
                            keep = (bmp[u][rx * 32 + ry] >> rz) & 1u;
                    }
                } else {
                    for (int u = 0; u < len && !keep; ++u) {
                        const int4 c = qc[u];
                        keep = max(abs(kc.x - c.x), max(abs(kc.y - c.y), abs(kc.z - c.z))) <= r;
                    }
                }
            }
        }
        // CTA-wide ordered compaction of `keep`
        const unsigned m = __ballot_sync(0xffffffffu, keep);
        if (lane == 0) wsum[wid] = __popc(m);
        __syncthreads();
        int before = 0, all = 0;
        for (int u = 0; u < nwarps; ++u) {
            before += u < wid ? wsum[u] : 0;
            all += wsum[u];
        }
        const int at = total + before + __popc(m & ((1u << lane) - 1));
        if (kFill && keep) wt_keys[out_base + at] = row;
        if (!kFill && keep && at < spill_cap) spill[(int64_t)t * spill_cap + at] = row;
        total += all;
        __syncthreads();
    }
    if (!kFill && threadIdx.x == 0) wt_cnt[t] = total;
}

// Runs of consecutive 8-row groups that cover each tile's window union (the attention kernel
// loads every run with one bulk copy). One warp per tile walks the ascending rows 32 at a time:
// a row opens a group when its group differs from the previous row's, and a group opens a run
// when it does not follow the previous group. kFill == false writes the run and group counts;
// kFill == true writes each run (first group, groups) at wr_off.
// The window key unions that fit their tile's spill slot, from the slot to wt_keys.
__global__ void k_copy_union(const int32_t* __restrict__ wt_off, const int32_t* __restrict__ spill,
                             int spill_cap, int32_t* __restrict__ wt_keys) {
    const int t = blockIdx.x;
    const int32_t a = wt_off[t], n = wt_off[t + 1] - a;
    if (n > spill_cap) return;
    for (int i = threadIdx.x; i < n; i += blockDim.x) wt_keys[a + i] = spill[(int64_t)t * spill_cap + i];
}

template <bool kFill>
__global__ void k_window_runs(int64_t T, const int32_t* __restrict__ wt_off,
                              const int32_t* __restrict__ wt_keys, int32_t* __restrict__ wr_cnt,
                              int32_t* __restrict__ wg_cnt, int32_t* __restrict__ wm_cnt,
                              const int32_t* __restrict__ wr_off, int2* __restrict__ runs) {
    const int lane = threadIdx.x & 31;
    const int64_t t = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const int32_t a = wt_off[t], b = wt_off[t + 1];
    const int32_t out = kFill ? wr_off[t] : 0;
    int32_t nr = 0, ng = 0, carry = -2;
    for (int32_t c = a; c < b; c += 32) {
        const int32_t i = c + lane;
        const bool valid = i < b;
        const int32_t gi = valid ? (wt_keys[i] >> 3) : 0x7fffffff;
        int32_t prev = __shfl_up_sync(0xffffffffu, gi, 1);
        if (lane == 0) prev = carry;
        const bool new_group = valid && gi != prev;
        const bool new_run = new_group && gi != prev + 1;
        const unsigned bg = __ballot_sync(0xffffffffu, new_group);
        const unsigned br = __ballot_sync(0xffffffffu, new_run);
        if (kFill && new_run) {
            // first group and, for now, the run's position in the group stream
            runs[out + nr + __popc(br & ((1u << lane) - 1u))] = make_int2(gi, ng + __popc(bg & ((1u << lane) - 1u)));
        }
        nr += __popc(br);
        ng += __popc(bg);
        const int last = min(31, b - 1 - c);
        carry = __shfl_sync(0xffffffffu, gi, last);
    }
    if (!kFill) {
        if (lane == 0) {
            wr_cnt[t] = nr;
            wg_cnt[t] = ng;
            wm_cnt[t] = (ng + 7) >> 3;
        }
        return;
    }
    __syncwarp();
    // group count of every run: the next run's stream position minus its own
    for (int32_t r = lane; r < nr; r += 32) {
        const int32_t nxt = r + 1 < nr ? runs[out + r + 1].y : ng;
        const int32_t cnt = nxt - runs[out + r].y;
        __syncwarp(__activemask());
        runs[out + r].y = cnt;
    }
}

// Window masks: for each query tile and each 64-key tile of its window stream (the runs' groups
// in order, 8 rows per group), bit c of row i says whether key c lies within Chebyshev distance r
// of query i. One thread per query row; key coordinates are read once per group by all threads.
__global__ void __launch_bounds__(kQTile) k_window_masks(const int32_t* __restrict__ qt_pos,
                                                         const int32_t* __restrict__ qt_len,
                                                         const int32_t* __restrict__ perm,
                                                         const int32_t* __restrict__ coords,
                                                         const int32_t* __restrict__ wr_off,
                                                         const int2* __restrict__ runs,
                                                         const int32_t* __restrict__ wm_off,
                                                         const int4* __restrict__ scoord, int r,
                                                         uint64_t* __restrict__ wmask) {
    const int t = blockIdx.x, row = threadIdx.x;
    const int32_t p0 = qt_pos[t], len = qt_len[t];
    const bool ok = row < len;
    int32_t qx = 0, qy = 0, qz = 0;
    if (ok) {
        const int32_t i = perm[p0 + row];
        qx = coords[3 * i];
        qy = coords[3 * i + 1];
        qz = coords[3 * i + 2];
    }
    uint64_t* out = wmask + (int64_t)wm_off[t] * kQTile + row;
    uint64_t word = 0;
    int q = 0;   // groups streamed so far
    for (int32_t ri = wr_off[t]; ri < wr_off[t + 1]; ++ri) {
        const int2 run = runs[ri];
        for (int32_t gi = run.x; gi < run.x + run.y; ++gi, ++q) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int4 kc = scoord[8 * (int64_t)gi + i];
                const int d = max(abs(kc.x - qx), max(abs(kc.y - qy), abs(kc.z - qz)));
                if (ok && d <= r) word |= 1ull << (((q & 7) << 3) + i);
            }
            if ((q & 7) == 7) {
                out[(int64_t)(q >> 3) * kQTile] = word;
                word = 0;
            }
        }
    }
    if (q & 7) out[(int64_t)(q >> 3) * kQTile] = word;
}

}  // namespace

#define SSA_ALLOC(ptr, type, count)                                                      \
    do {                                                                                 \
        ptr = (type*)plan_alloc(p, sizeof(type) * (size_t)std::max<int64_t>((count), 1)); \
        if (!ptr) return SSA_ERR_ALLOC;                                                  \
    } while (0)

ssa_status_t build_plan(Plan* p, const int32_t* coords, cudaStream_t st) {
    const int64_t N = p->N;
    const int B = p->B;
    const int r = p->r;
    // ---- constants ---------------------------------------------------------------------------
    SSA_ALLOC(p->d_seqs, SeqInfo, B);
    SSA_ALLOC(p->d_status, int32_t, 1);
    SSA_ALLOC(p->coords, int32_t, 3 * N);
    if (cudaMemcpyAsync(p->d_seqs, p->seqs.data(), sizeof(SeqInfo) * B, cudaMemcpyHostToDevice, st) ||
        cudaMemcpyAsync(p->coords, coords, sizeof(int32_t) * 3 * N, cudaMemcpyDeviceToDevice, st) ||
        cudaMemsetAsync(p->d_status, 0, sizeof(int32_t), st))
        return SSA_ERR_CUDA;

    const int64_t G = p->G;
    const int64_t cap_mb = std::min<int64_t>(G, N);
    uint64_t hsize = 1024;
    while (hsize < (uint64_t)(2 * N)) hsize <<= 1;
    int64_t tmp_len = scan_tmp_len(std::max<int64_t>(G, N) + 1);

    int32_t *tok_key, *key_cnt, *bidx, *key2blk, *blk_cnt, *blk_pcnt, *tmp, *blk_fill;
    uint64_t* hkeys;
    int32_t* hvals;
    SSA_ALLOC(tok_key, int32_t, N);
    SSA_ALLOC(key_cnt, int32_t, G);
    SSA_ALLOC(bidx, int32_t, G + 1);
    SSA_ALLOC(key2blk, int32_t, G);
    SSA_ALLOC(blk_cnt, int32_t, cap_mb + 1);
    SSA_ALLOC(blk_pcnt, int32_t, cap_mb + 1);
    SSA_ALLOC(blk_fill, int32_t, cap_mb + 1);
    SSA_ALLOC(tmp, int32_t, tmp_len);
    SSA_ALLOC(hkeys, uint64_t, hsize);
    SSA_ALLOC(hvals, int32_t, hsize);
    SSA_ALLOC(p->blk_off, int32_t, cap_mb + 1);
    SSA_ALLOC(p->blk_poff, int32_t, cap_mb + 1);
    SSA_ALLOC(p->blk_coord, int32_t, 3 * cap_mb);
    SSA_ALLOC(p->blk_seq, int32_t, cap_mb);
    if (cudaMemsetAsync(key_cnt, 0, sizeof(int32_t) * G, st) ||
        cudaMemsetAsync(blk_cnt, 0, sizeof(int32_t) * (cap_mb + 1), st) ||
        cudaMemsetAsync(blk_pcnt, 0, sizeof(int32_t) * (cap_mb + 1), st) ||
        cudaMemsetAsync(blk_fill, 0, sizeof(int32_t) * (cap_mb + 1), st) ||
        cudaMemsetAsync(hkeys, 0xff, sizeof(uint64_t) * hsize, st))
        return SSA_ERR_CUDA;

    // ---- a1: keys, histogram, hash -------------------------------------------------------------
    k_keys_and_hash<<<grid_for(N), kThreads, 0, st>>>(coords, N, p->d_seqs, B, tok_key, key_cnt,
                                                      hkeys, hvals, hsize - 1, p->d_status);
    k_occupied<<<grid_for(G), kThreads, 0, st>>>(key_cnt, G, bidx);
    trace_step("plan keys+hash", st);
    note_launch(2);
    scan_exclusive(bidx, bidx, G, tmp, st);
    k_blocks<<<grid_for(G), kThreads, 0, st>>>(key_cnt, bidx, G, p->d_seqs, B, key2blk, blk_cnt,
                                               blk_pcnt, p->blk_coord, p->blk_seq);
    note_launch();
    scan_exclusive(blk_cnt, p->blk_off, cap_mb, tmp, st);
    scan_exclusive(blk_pcnt, p->blk_poff, cap_mb, tmp, st);
    trace_step("plan blocks", st);

    // ---- a2: the per-token neighbour counts and lists are built on first use --------------------
    const int cube = (2 * r + 1) * (2 * r + 1) * (2 * r + 1);
    int cap = 32;
    while (cap < cube) cap <<= 1;

    // ---- first wait: sizes and coordinate errors --------------------------------------------------
    int32_t h_sizes[4];
    if (cudaMemcpyAsync(&h_sizes[0], bidx + G, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaMemcpyAsync(&h_sizes[1], p->blk_poff + cap_mb, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaMemcpyAsync(&h_sizes[3], p->d_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    if (h_sizes[3] & DEV_COORD_RANGE) return SSA_ERR_COORD_RANGE;
    if (h_sizes[3] & DEV_DUPLICATE) return SSA_ERR_DUPLICATE_COORD;
    if (h_sizes[3]) return SSA_ERR_CUDA;
    p->Mb = h_sizes[0];
    p->Npad = h_sizes[1];
    p->nnz = -1;   // counted on first use

    // ---- a1: scatter, per-block sort, positions ------------------------------------------------
    SSA_ALLOC(p->perm, int32_t, N);
    SSA_ALLOC(p->tok_blk, int32_t, N);
    SSA_ALLOC(p->tok_pos, int32_t, N);
    SSA_ALLOC(p->spos_tok, int32_t, p->Npad);
    SSA_ALLOC(p->scoord, int4, p->Npad);
    SSA_ALLOC(p->blk_info, int2, p->Mb);
    k_block_info<<<grid_for(p->Mb), kThreads, 0, st>>>(p->blk_off, p->blk_poff, p->Mb, p->blk_info);
    note_launch();
    k_scatter<<<grid_for(N), kThreads, 0, st>>>(tok_key, key2blk, N, p->blk_off, blk_fill, p->perm,
                                                p->tok_blk);
    k_sort_blocks<<<grid_for(p->Mb, 8), 256, 0, st>>>(p->perm, p->blk_off, p->Mb);
    k_fill_i32<<<grid_for(p->Npad), kThreads, 0, st>>>(p->spos_tok, p->Npad, -1);
    // padding rows sit far outside every grid so no window test ever accepts them
    k_fill_int4<<<grid_for(p->Npad), kThreads, 0, st>>>(p->scoord, p->Npad,
                                                        make_int4(1 << 28, 1 << 28, 1 << 28, -1));
    k_positions<<<grid_for(N), kThreads, 0, st>>>(p->perm, p->tok_blk, p->blk_off, p->blk_poff,
                                                  p->coords, N, p->tok_pos, p->spos_tok, p->scoord);
    trace_step("plan scatter/sort/positions", st);
    note_launch(5);

    // ---- a2: the per-token neighbour lists are built on first use (ensure_neighbours) ----------------
    p->hkeys = hkeys;
    p->hvals = hvals;
    p->hmask = hsize - 1;
    p->nbr_cap = cap;
    p->nbr_idx = nullptr;
    p->blk_nbr = nullptr;   // block neighbour table (convolution compression), built on first use
    p->sb_rows = nullptr;   // sub-block order and selection tiles (shared selection), first use
    p->sst = nullptr;
    p->n_sst = 0;

    // ---- query tiles and their window key unions (tensor-core window kernel) ----------------------
    std::vector<int32_t> qpos, qlen, qseq;
    for (int s = 0; s < B; ++s) {
        for (int64_t a = p->seqs[s].lo; a < p->seqs[s].hi; a += kQTile) {
            qpos.push_back((int32_t)a);
            qlen.push_back((int32_t)std::min<int64_t>(kQTile, p->seqs[s].hi - a));
            qseq.push_back(s);
        }
    }
    p->n_qtiles = (int64_t)qpos.size();
    const int64_t T = p->n_qtiles;
    SSA_ALLOC(p->qt_pos, int32_t, T);
    SSA_ALLOC(p->qt_len, int32_t, T);
    SSA_ALLOC(p->qt_seq, int32_t, T);
    SSA_ALLOC(p->wt_off, int32_t, T + 1);
    if (cudaMemcpyAsync(p->qt_pos, qpos.data(), sizeof(int32_t) * T, cudaMemcpyHostToDevice, st) ||
        cudaMemcpyAsync(p->qt_len, qlen.data(), sizeof(int32_t) * T, cudaMemcpyHostToDevice, st) ||
        cudaMemcpyAsync(p->qt_seq, qseq.data(), sizeof(int32_t) * T, cudaMemcpyHostToDevice, st))
        return SSA_ERR_CUDA;
    int32_t *wt_cnt, *spill;
    SSA_ALLOC(wt_cnt, int32_t, T + 1);
    // One pass finds each tile's window union; unions of up to spill_cap rows are kept in a slot
    // per tile (at most 256 MB in all) and copied once their offsets are known, larger ones are
    // found again by a second pass that skips every other tile.
    int spill_cap = (int)std::min<int64_t>(4096, ((int64_t)64 << 20) / std::max<int64_t>(T, 1));
    spill_cap = spill_cap >= 256 ? spill_cap & ~31 : 0;
    SSA_ALLOC(spill, int32_t, (int64_t)T * std::max(spill_cap, 1));
    k_window_union<false><<<(unsigned)T, 128, 0, st>>>(
        p->qt_pos, p->qt_len, p->qt_seq, p->perm, p->tok_blk, p->coords, p->blk_coord, p->blk_poff,
        p->blk_off, key2blk, p->d_seqs, p->scoord, r, wt_cnt, nullptr, nullptr, spill, spill_cap);
    note_launch();
    trace_step("plan neighbour lists + window union counts", st);
    scan_exclusive(wt_cnt, p->wt_off, T, tmp, st);
    int32_t n_wkeys = 0;
    if (cudaMemcpyAsync(&n_wkeys, p->wt_off + T, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    if (n_wkeys < 0) return SSA_ERR_UNSUPPORTED;
    SSA_ALLOC(p->wt_keys, int32_t, n_wkeys);
    k_copy_union<<<(unsigned)T, 128, 0, st>>>(p->wt_off, spill, spill_cap, p->wt_keys);
    k_window_union<true><<<(unsigned)T, 128, 0, st>>>(
        p->qt_pos, p->qt_len, p->qt_seq, p->perm, p->tok_blk, p->coords, p->blk_coord, p->blk_poff,
        p->blk_off, key2blk, p->d_seqs, p->scoord, r, nullptr, p->wt_off, p->wt_keys, nullptr, spill_cap);
    note_launch(2);
    trace_step("plan window unions", st);
    int32_t *wr_cnt, *wm_cnt;
    SSA_ALLOC(wr_cnt, int32_t, T + 1);
    SSA_ALLOC(wm_cnt, int32_t, T + 1);
    SSA_ALLOC(p->wr_off, int32_t, T + 1);
    SSA_ALLOC(p->wg_cnt, int32_t, T);
    SSA_ALLOC(p->wm_off, int32_t, T + 1);
    k_window_runs<false><<<(unsigned)cdiv(T, 4), 128, 0, st>>>(T, p->wt_off, p->wt_keys, wr_cnt,
                                                                p->wg_cnt, wm_cnt, nullptr, nullptr);
    note_launch();
    scan_exclusive(wr_cnt, p->wr_off, T, tmp, st);
    scan_exclusive(wm_cnt, p->wm_off, T, tmp, st);

    // block range of every sequence (host copy for launches)
    p->seq_blk.assign(B + 1, 0);
    std::vector<int32_t> sb(B + 1);
    for (int s = 0; s <= B; ++s) {
        int64_t key = s < B ? p->seqs[s].dense_base : G;
        if (cudaMemcpyAsync(&sb[s], bidx + key, sizeof(int32_t), cudaMemcpyDeviceToHost, st))
            return SSA_ERR_CUDA;
    }
    int32_t status = 0, n_runs = 0, n_wtiles = 0;
    if (cudaMemcpyAsync(&status, p->d_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaMemcpyAsync(&n_runs, p->wr_off + T, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaMemcpyAsync(&n_wtiles, p->wm_off + T, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    SSA_ALLOC(p->wr_runs, int2, n_runs);
    SSA_ALLOC(p->wmask, uint64_t, (int64_t)n_wtiles * kQTile);
    k_window_runs<true><<<(unsigned)cdiv(T, 4), 128, 0, st>>>(T, p->wt_off, p->wt_keys, nullptr,
                                                               nullptr, nullptr, p->wr_off, p->wr_runs);
    k_window_masks<<<(unsigned)T, kQTile, 0, st>>>(p->qt_pos, p->qt_len, p->perm, p->coords, p->wr_off,
                                                   p->wr_runs, p->wm_off, p->scoord, r, p->wmask);
    note_launch(2);
    trace_step("plan window runs + masks", st);
    for (int s = 0; s <= B; ++s) p->seq_blk[s] = sb[s];
    SSA_ALLOC(p->seq_blk_d, int32_t, B + 1);
    if (cudaMemcpyAsync(p->seq_blk_d, sb.data(), sizeof(int32_t) * (B + 1), cudaMemcpyHostToDevice, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    if (status) return SSA_ERR_CUDA;

    // ---- pools of small blocks: per sequence, after all padded block rows -------------------------
    int32_t* ptok;
    SSA_ALLOC(p->blk_tpool, int32_t, std::max<int64_t>(p->Mb, 1));
    SSA_ALLOC(ptok, int32_t, B);
    k_tiny_pool<<<(unsigned)B, 256, 0, st>>>(p->blk_off, p->seq_blk_d, p->blk_tpool, ptok);
    note_launch();
    std::vector<int32_t> hp(B);
    if (cudaMemcpyAsync(hp.data(), ptok, sizeof(int32_t) * B, cudaMemcpyDeviceToHost, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    std::vector<int2> sp(B);
    int64_t pg = p->Npad / 8;
    for (int s = 0; s < B; ++s) {
        const int32_t groups = (hp[s] + 7) / 8;
        sp[s] = make_int2((int32_t)pg, groups);
        pg += groups;
    }
    p->Nks = 8 * pg;
    SSA_ALLOC(p->seq_pool, int2, B);
    if (cudaMemcpyAsync(p->seq_pool, sp.data(), sizeof(int2) * B, cudaMemcpyHostToDevice, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;

    // scratch of the plan build is released now
    void* scratch[] = {tok_key, key_cnt, bidx, key2blk, blk_cnt, blk_pcnt, blk_fill,
                       tmp, wt_cnt, wr_cnt, wm_cnt, ptok, spill};
    for (void* ptr : scratch) {
        auto it = std::find(p->owned.begin(), p->owned.end(), ptr);
        if (it != p->owned.end()) {
            p->release(ptr, st, p->alloc_ctx);
            p->owned.erase(it);
        }
    }
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

// ---- sub-block order and selection tiles (selection shared by a 4x4x4 sub-block) ----------------
// One warp per block. A token's sub-block within its block is the 3-bit index of
// ((x >> 2) & 1, (y >> 2) & 1, (z >> 2) & 1) (4 divides 8, so a sub-block never leaves its block).
// Writes the block's sorted positions grouped by sub-block (stable) to sb_rows, and the tokens of
// each of its 8 sub-blocks to sbc[8 b + s].
__global__ void k_subblock_order(const int32_t* __restrict__ perm, const int32_t* __restrict__ coords,
                                 const int32_t* __restrict__ blk_off, int32_t* __restrict__ sb_rows,
                                 int32_t* __restrict__ sbc) {
    const int b = blockIdx.x, lane = threadIdx.x;
    const int32_t a0 = blk_off[b], n = blk_off[b + 1] - a0;
    auto sub_of = [&](int32_t pos) {
        const int32_t* c = coords + 3 * (int64_t)perm[pos];
        return (((c[0] >> 2) & 1) << 2) | (((c[1] >> 2) & 1) << 1) | ((c[2] >> 2) & 1);
    };
    int mine = 0;   // lane s < 8: tokens of sub-block s
    for (int i = 0; i < n; i += 32) {
        const int s = i + lane < n ? sub_of(a0 + i + lane) : -1;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const unsigned bal = __ballot_sync(0xffffffffu, s == q);
            if (lane == q) mine += __popc(bal);
        }
    }
    int base = mine;   // exclusive prefix over lanes 0..7
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, base, d);
        if (lane >= d) base += t;
    }
    base -= mine;
    if (lane < 8) sbc[8 * (int64_t)b + lane] = mine;
    for (int i = 0; i < n; i += 32) {
        const int s = i + lane < n ? sub_of(a0 + i + lane) : -1;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const unsigned bal = __ballot_sync(0xffffffffu, s == q);
            const int bq = __shfl_sync(0xffffffffu, base, q);
            if (s == q) sb_rows[a0 + bq + __popc(bal & ((1u << lane) - 1u))] = a0 + i + lane;
            if (lane == q) base += __popc(bal);
        }
    }
}

ssa_status_t ensure_subblock_tiles(Plan* p, cudaStream_t st) {
    if (p->sst) return SSA_OK;
    if (p->Mb == 0) {
        SSA_ALLOC(p->sst, int4, 1);
        p->n_sst = 0;
        return SSA_OK;
    }
    int32_t* sbc;
    SSA_ALLOC(p->sb_rows, int32_t, p->N);
    SSA_ALLOC(sbc, int32_t, 8 * p->Mb);
    k_subblock_order<<<(unsigned)p->Mb, 32, 0, st>>>(p->perm, p->coords, p->blk_off, p->sb_rows, sbc);
    note_launch();
    std::vector<int32_t> cnt((size_t)(8 * p->Mb)), off((size_t)(p->Mb + 1));
    if (cudaMemcpyAsync(cnt.data(), sbc, sizeof(int32_t) * cnt.size(), cudaMemcpyDeviceToHost, st) ||
        cudaMemcpyAsync(off.data(), p->blk_off, sizeof(int32_t) * off.size(), cudaMemcpyDeviceToHost, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    // Tiles take the sub-blocks of a sequence in order (blocks in order, sub-blocks within), a new
    // tile whenever the next sub-block would pass 128 rows or 32 sub-blocks (a sub-block has at
    // most 64 rows). Tile = (first index into sb_rows, rows, sequence, sub-blocks).
    std::vector<int4> tiles;
    for (int32_t s = 0; s < p->B; ++s) {
        int32_t first = 0, rows = 0, nsub = 0;
        for (int64_t b = p->seq_blk[s]; b < p->seq_blk[s + 1]; ++b) {
            int32_t at = off[b];
            for (int q = 0; q < 8; ++q) {
                const int32_t c = cnt[8 * b + q];
                if (c == 0) continue;
                if (rows > 0 && (rows + c > 128 || nsub == 32)) {
                    tiles.push_back(make_int4(first, rows, s, nsub));
                    rows = 0;
                    nsub = 0;
                }
                if (rows == 0) first = at;
                rows += c;
                nsub += 1;
                at += c;
            }
        }
        if (rows > 0) tiles.push_back(make_int4(first, rows, s, nsub));
    }
    p->n_sst = (int64_t)tiles.size();
    SSA_ALLOC(p->sst, int4, std::max<int64_t>(p->n_sst, 1));
    if (p->n_sst > 0 &&
        (cudaMemcpyAsync(p->sst, tiles.data(), sizeof(int4) * tiles.size(), cudaMemcpyHostToDevice, st) ||
         cudaStreamSynchronize(st)))
        return SSA_ERR_CUDA;
    auto it = std::find(p->owned.begin(), p->owned.end(), (void*)sbc);
    if (it != p->owned.end()) {
        p->release(sbc, st, p->alloc_ctx);
        p->owned.erase(it);
    }
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

ssa_status_t ensure_neighbour_counts(Plan* p, cudaStream_t st) {
    if (p->nnz >= 0) return SSA_OK;
    const int cap = p->nbr_cap;
    const int warps = std::max(1, std::min(8, 8192 / cap));
    int32_t *cnt, *tmp;
    SSA_ALLOC(p->nbr_off32, int32_t, p->N + 1);
    SSA_ALLOC(cnt, int32_t, p->N + 1);
    SSA_ALLOC(tmp, int32_t, scan_tmp_len(p->N + 1));
    k_neighbours<false><<<grid_for(p->N, warps), warps * 32, 0, st>>>(
        p->coords, p->N, p->d_seqs, p->B, p->r, p->hkeys, p->hvals, p->hmask, cnt, nullptr, nullptr,
        cap, p->d_status);
    note_launch();
    scan_exclusive(cnt, p->nbr_off32, p->N, tmp, st);
    int32_t total = 0;
    if (cudaMemcpyAsync(&total, p->nbr_off32 + p->N, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    for (void* ptr : {(void*)cnt, (void*)tmp}) {
        auto it = std::find(p->owned.begin(), p->owned.end(), ptr);
        if (it != p->owned.end()) {
            p->release(ptr, st, p->alloc_ctx);
            p->owned.erase(it);
        }
    }
    if (total < 0) return SSA_ERR_UNSUPPORTED;   // more than 2^31 neighbour pairs
    p->nnz = total;
    return SSA_OK;
}

ssa_status_t ensure_neighbours(Plan* p, cudaStream_t st) {
    ssa_status_t rc = ensure_neighbour_counts(p, st);
    if (rc != SSA_OK) return rc;
    if (p->nbr_idx || p->nnz == 0) return SSA_OK;
    SSA_ALLOC(p->nbr_idx, int32_t, p->nnz);
    const int cap = p->nbr_cap;
    const int warps = std::max(1, std::min(8, 8192 / cap));
    k_neighbours<true><<<grid_for(p->N, warps), warps * 32, (size_t)warps * cap * sizeof(int32_t), st>>>(
        p->coords, p->N, p->d_seqs, p->B, p->r, p->hkeys, p->hvals, p->hmask, nullptr, p->nbr_off32,
        p->nbr_idx, cap, p->d_status);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

}  // namespace ssa
