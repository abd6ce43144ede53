// Internal definitions shared by the translation units of libssa.so.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <vector>

#include "../../include/ssa.h"

namespace ssa {

// Bits of the device status word (one int32 per plan). Kernels OR these in; the host maps them to
// ssa_status_t when it next waits for the device.
enum : int32_t {
    DEV_COORD_RANGE = 1,
    DEV_DUPLICATE = 2,
    DEV_TIMEOUT = 4,
    DEV_BAD_INDEX = 8,
    DEV_TOO_LARGE = 16,
};

constexpr int kBlockEdge = 8;      // block edge in voxels (the only supported value)
constexpr int kPad = 8;            // blocks start on multiples of 8 rows (one group) in the K/V copies
constexpr int kQTile = 128;        // query rows per tensor-core tile
constexpr int kMaxTopk = 32;
// blocks of at most this many tokens (less than one 8-row group) also get a packed copy in
// their sequence's pool, which the selected branch may stream in their place
constexpr int kPoolMaxTokens = 7;

// Per-sequence constants, mirrored on the device.
struct SeqInfo {
    int64_t lo, hi;          // token range [lo, hi)
    int64_t dense_base;      // first dense block key of this sequence
    int32_t gx, gy, gz;      // grid extent
    int32_t gbx, gby, gbz;   // blocks per axis (ceil(g / 8))
};

// Attention prologue of a forward call: RMS normalisation of q and k over the head dimension
// (weights q_gamma, k_gamma: device fp32 [D]) and the 3D rotary embedding with base theta at the
// voxel coordinates (prologue.cuh). Off when q_gamma is null.
struct Prologue {
    const float* q_gamma = nullptr;
    const float* k_gamma = nullptr;
    double theta = 10000.0;
    float eps = 1e-6f;
    bool on() const { return q_gamma != nullptr; }
};

// Forward workspace, cached in the plan for one (H, D, dtype, k).
struct Workspace {
    int32_t H = 0, D = 0, k = 0;
    ssa_dtype_t dtype = SSA_F32;
    // K_s, V_s: per head, the K / V rows in padded block order (Npad rows) followed by each
    // sequence's pool of small blocks (their rows again, packed), stored as 8-row groups in the
    // tensor cores' swizzled operand order (see pool.cu); padding rows are zero.
    void* ks = nullptr;        // [H, Nks, D] T
    void* vs = nullptr;        // [H, Nks, D] T
    void* kc = nullptr;        // [H, Mb, D]   T (fp32 for the fp32 path), row-major
    void* vc = nullptr;        // [H, Mb, D]
    void* kcg = nullptr;       // [H, Mb8, D]  T   compressed tokens in the grouped order (16-bit path)
    void* vcg = nullptr;       // [H, Mb8, D]
    int64_t Mb8 = 0;           // Mb rounded up to a multiple of 8
    float* base = nullptr;     // [query tiles, H, D/4, 128, 4] running g0*o_cmp + g1*o_sel
    int32_t* sel = nullptr;    // [N, H, k]        selected blocks, sorted token order
    // fp32 path with the prologue: transformed q and k (allocated on first use)
    float* qp = nullptr;       // [N, H, D]
    float* kp = nullptr;       // [N, H, D]
    // convolution compression and predicted gates (allocated on first use)
    float* means = nullptr;    // [2][H][Mb][D] block means of K and V
    float* gates = nullptr;    // [N, H, 3] predicted gates
    // host-buffer entry point staging (allocated on first use)
    void* h_q = nullptr; void* h_k = nullptr; void* h_v = nullptr; void* h_out = nullptr;
    float* h_gates = nullptr; float* h_wc = nullptr;
    std::vector<void*> owned;
};

// Host-buffer entry point, heads in chunks: copies in (s_in), the forward of a chunk (the
// caller's stream) and copies out (s_out) overlap; two slots of device buffers.
struct HostPipe {
    int32_t hc = 0;                 // heads per chunk the buffers are sized for (0 = none yet)
    int32_t H = 0, D = 0;
    ssa_dtype_t dtype = SSA_F32;
    cudaStream_t s_in = nullptr, s_out = nullptr;
    cudaEvent_t e_in[2] = {nullptr, nullptr}, e_comp[2] = {nullptr, nullptr}, e_out[2] = {nullptr, nullptr};
    cudaEvent_t e_par = nullptr;    // gates and Wc copied
    cudaEvent_t e_start = nullptr;  // the caller's stream at entry
    void* q[2] = {nullptr, nullptr};
    void* k[2] = {nullptr, nullptr};
    void* v[2] = {nullptr, nullptr};
    void* o[2] = {nullptr, nullptr};
    float* g[2] = {nullptr, nullptr};
    float* gates = nullptr;         // [N, H, 3] all heads
    float* wc = nullptr;            // [D, D]
    std::vector<void*> owned;
};

struct Plan {
    int device = 0;
    cudaStream_t stream = nullptr;  // creation stream (frees are queued here)
    ssa_alloc_fn alloc = nullptr;
    ssa_free_fn release = nullptr;
    void* alloc_ctx = nullptr;

    int64_t N = 0;
    int32_t B = 0;
    int32_t r = 0;
    int64_t G = 0;       // dense block keys over all sequences
    int64_t Mb = 0;      // occupied blocks
    int64_t Npad = 0;    // padded sorted rows
    int64_t Nks = 0;     // rows per head of K_s / V_s: the Npad padded rows, then the pools
    int64_t nnz = -1;    // window neighbour pairs (-1 until counted on first use)
    int64_t n_qtiles = 0;
    std::vector<SeqInfo> seqs;
    std::vector<int64_t> seq_blk;   // [B+1] block range of each sequence (host copy)

    SeqInfo* d_seqs = nullptr;
    int32_t* d_status = nullptr;
    int32_t* coords = nullptr;   // [N,3] copy of the input coordinates
    int32_t* perm = nullptr;     // [N]
    int32_t* tok_blk = nullptr;  // [N]
    int32_t* tok_pos = nullptr;  // [N]  position in perm
    int32_t* blk_off = nullptr;  // [Mb+1]
    int32_t* blk_poff = nullptr; // [Mb+1] padded row offsets
    int2* blk_info = nullptr;    // [Mb] (first 8-row group of the padded rows, tokens)
    int32_t* blk_tpool = nullptr;// [Mb] row of a small block's copy in its sequence's pool
                                 //      (relative to the pool's first row), -1 for other blocks
    int2* seq_pool = nullptr;    // [B] (first 8-row group, groups) of each sequence's pool
    int32_t* blk_coord = nullptr;// [Mb,3]
    int32_t* blk_seq = nullptr;  // [Mb]
    int32_t* seq_blk_d = nullptr;// [B+1]
    int32_t* spos_tok = nullptr; // [Npad] token of each padded row, -1 for padding
    int4* scoord = nullptr;      // [Npad] (x, y, z, block) of each padded row; padding far away
    int32_t* nbr_off32 = nullptr;// [N+1]
    int32_t* nbr_idx = nullptr;  // [nnz], built on first use (backward, export): the forward's
                                 // window runs and masks do not need per-token lists
    uint64_t* hkeys = nullptr;   // coordinate hash (kept for the lazy neighbour lists)
    int32_t* hvals = nullptr;
    uint64_t hmask = 0;
    int32_t nbr_cap = 32;        // per-warp sort buffer of the neighbour-list kernel
    int32_t* blk_nbr = nullptr;  // [Mb][27] block at offset o of every block (-1 = none), first use
    int32_t* sb_rows = nullptr;  // [N] sorted positions, each block's tokens in 4x4x4 sub-block
                                 //      order (then ascending position); first use of shared selection
    int4* sst = nullptr;         // [n_sst] selection tiles of whole sub-blocks of one sequence:
                                 //      (first index into sb_rows, rows <= 128, sequence, sub-blocks <= 32)
    int64_t n_sst = 0;
    int32_t* qt_pos = nullptr;   // [n_qtiles] first sorted position of each query tile
    int32_t* qt_len = nullptr;   // [n_qtiles]
    int32_t* qt_seq = nullptr;   // [n_qtiles]
    int32_t* wt_off = nullptr;   // [n_qtiles+1] window key union per query tile (CSR)
    int32_t* wt_keys = nullptr;  // padded rows, ascending
    int32_t* wr_off = nullptr;   // [n_qtiles+1] runs of consecutive 8-row groups covering wt_keys (CSR)
    int2* wr_runs = nullptr;     // (first group, groups) of each run
    int32_t* wg_cnt = nullptr;   // [n_qtiles] groups of each tile's window union
    int32_t* wm_off = nullptr;   // [n_qtiles+1] first 64-key window tile of each query tile
    uint64_t* wmask = nullptr;   // [wm_off[T]][128] window mask: bit c of row i = key c within r
    std::vector<void*> owned;
    Workspace ws;
    Workspace ws_chunk;   // workspace of the chunked host-buffer path (its heads per chunk)
    HostPipe hp;
    void* cublas = nullptr;   // cuBLAS handle of the backward's compressed-branch GEMMs (first use)
};

extern std::atomic<int64_t> g_launches;
inline void note_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }
// Opt-in launch trace (environment variable SSA_TRACE=1): waits for `st` after the named step
// and reports it on stderr with its duration. Off by default; used to locate a stuck kernel.
void trace_step(const char* what, cudaStream_t st);

// Opt-in kernel timing (ssa_profile_enable): a ProfScope brackets one launch with CUDA events on
// the launch stream; ssa_profile_read accumulates the durations per kernel name.
bool profiling_on();
void profile_record(const char* name, cudaEvent_t start, cudaEvent_t stop);
cudaEvent_t profile_event();
struct ProfScope {
    const char* name;
    cudaStream_t st;
    cudaEvent_t a = nullptr;
    ProfScope(const char* n, cudaStream_t s) : name(n), st(s) {
        if (profiling_on()) {
            a = profile_event();
            cudaEventRecord(a, st);
        }
    }
    ~ProfScope() {
        if (a) {
            cudaEvent_t b = profile_event();
            cudaEventRecord(b, st);
            profile_record(name, a, b);
        }
    }
};

// ---- allocation through the plan's hook -------------------------------------------------------
void* plan_alloc(Plan* p, size_t bytes);
void plan_free_all(Plan* p, std::vector<void*>& list);

// ---- launchers implemented in the .cu files ---------------------------------------------------
// scan.cu: out[i] = sum_{t<i} in[t] for i in [0, n], out[n] = total. `tmp` holds scan_tmp_len(n)
// ints. In-place (out == in) is allowed.
int64_t scan_tmp_len(int64_t n);
void scan_exclusive(const int32_t* in, int32_t* out, int64_t n, int32_t* tmp, cudaStream_t s);

// plan.cu
ssa_status_t build_plan(Plan* p, const int32_t* coords, cudaStream_t s);
// the per-token window neighbour counts (nbr_off32, nnz) and lists (nbr_idx), built once per plan
// on first use (fp32 forward, backward, export, size query)
ssa_status_t ensure_neighbour_counts(Plan* p, cudaStream_t s);
ssa_status_t ensure_neighbours(Plan* p, cudaStream_t s);

// pool.cu (with the prologue applied to k on the way when pro.on(), 16-bit types). With `means`
// non-null: writes the fp32 block means [2][H][Mb][D] (K, then V) instead of the compressed tokens.
void launch_pool(const Plan* p, const Workspace& w, const void* k, const void* v, const float* wc,
                 const Prologue& pro, float* means, cudaStream_t s);

// conv.cu: compressed tokens by the sparse 3D convolution over the block grid from the block
// means (w.kc/w.vc, and the grouped copies for 16-bit types); the 27 neighbours of every block.
ssa_status_t ensure_block_neighbours(Plan* p, cudaStream_t s);
void launch_conv_compress(const Plan* p, const Workspace& w, const float* means, const float* wconv,
                          cudaStream_t s);
// gates [N, H, 3] = sigmoid(q . wg + bg) for fp32 q (the 16-bit path predicts them in select.cu)
void launch_gates_f32(const Plan* p, const float* q, const float* wg, const float* bg, int H, int D,
                      float* gates, cudaStream_t s);

// prologue.cu: out = prologue(x) for fp32 [N, H, D] rows (the fp32 path's stand-alone pass)
void launch_qk_prologue_f32(const Plan* p, const float* x, const float* gamma, const Prologue& pro,
                            int H, int D, float* out, cudaStream_t s);

// Per-branch outputs of the forward, fp32 [N, H, D] in token order each: o_cmp, o_sel, o_win
// (normalised branch attention outputs before the gates). Any entry may be null.
struct BranchOut {
    float* o[3] = {nullptr, nullptr, nullptr};
};

// attn_simt.cu (fp32 path)
void launch_forward_simt(const Plan* p, const Workspace& w, const void* q, const void* k,
                         const void* v, const float* gates, void* out, const BranchOut& bo,
                         cudaStream_t s);

// select.cu (bf16 / fp16 path): the selected blocks of every (token, head) into w.sel, sorted
// token order (the prologue, when on, is applied to each query tile after it is loaded)
// With gate_w non-null it also writes gates_out [N, H, 3] = sigmoid(q . gate_w + gate_b), q being the
// query as the attention sees it (after the prologue).
ssa_status_t ensure_subblock_tiles(Plan* p, cudaStream_t st);
ssa_status_t launch_select_shared(const Plan* p, const Workspace& w, const void* q, const Prologue& pro,
                                  const float* gate_w, const float* gate_b, float* gates_out,
                                  cudaStream_t st);
ssa_status_t launch_select_tc(const Plan* p, const Workspace& w, const void* q, const Prologue& pro,
                              const float* gate_w, const float* gate_b, float* gates_out, cudaStream_t s);

// attn_fwd.cu (bf16 / fp16 path): the fused tensor-core forward over w.sel (the prologue, when on, is
// applied to each query tile after it is loaded)
ssa_status_t launch_forward_tc(const Plan* p, const Workspace& w, const void* q, const float* gates,
                               void* out, const BranchOut& bo, const Prologue& pro, cudaStream_t s);

// backward.cu
void destroy_blas(Plan* p);
ssa_status_t launch_backward(Plan* p, const Workspace& w, const void* q, const void* k,
                             const void* v, const float* gates, const float* wc, const void* dout,
                             void* dq, void* dk, void* dv, cudaStream_t s);

// selftest.cu: a bounded wait on an mbarrier nothing arrives at (records DEV_TIMEOUT)
ssa_status_t launch_wait_timeout(Plan* p, int64_t max_cycles, cudaStream_t s);

// selection export (attn_fwd.cu): sel_out [N,H,k] in token order from the sorted-order buffer.
void launch_export_sel(const Plan* p, const Workspace& w, int32_t* sel_out, cudaStream_t s);

// ---- small device helpers -------------------------------------------------------------------
__host__ __device__ inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline int64_t round_up(int64_t a, int64_t b) { return cdiv(a, b) * b; }

template <typename T> struct Elem;
template <> struct Elem<float> {
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__half> {
    static __device__ __forceinline__ float to_f(__half x) { return __half2float(x); }
    static __device__ __forceinline__ __half from_f(float x) { return __float2half_rn(x); }
};
template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// Byte offset of element column d (a multiple of 8) of row `row` of a grouped matrix with D
// columns of a 16-bit type: rows go 8 at a time; a group stores its D/32 column chunks as 512-byte
// atoms of 8 rows x 64 bytes whose 16-byte units of row i are permuted by unit ^= (i >> 1) & 3
// (the tensor cores' shared-memory operand order with 64-byte swizzle).
__device__ __forceinline__ int64_t grouped_off(int64_t row, int d, int D) {
    const int64_t g = row >> 3;
    const int i = (int)(row & 7), c = d >> 5, u = (d & 31) >> 3;
    return g * (int64_t)(D / 32) * 512 + c * 512 + i * 64 + ((u ^ ((i >> 1) & 3)) << 4);
}

// Packed (sequence, x, y, z) key of the coordinate hash; each field < 2^16.
__device__ __forceinline__ uint64_t pack_cell(int32_t s, int32_t x, int32_t y, int32_t z) {
    return ((uint64_t)(uint32_t)s << 48) | ((uint64_t)(uint32_t)x << 32) |
           ((uint64_t)(uint32_t)y << 16) | (uint64_t)(uint32_t)z;
}
// MurmurHash3 64-bit finaliser: spreads packed keys over the table.
__device__ __forceinline__ uint64_t mix64(uint64_t k) {
    k ^= k >> 33;
    k *= 0xff51afd7ed558ccdULL;
    k ^= k >> 33;
    k *= 0xc4ceb9fe1a85ec53ULL;
    k ^= k >> 33;
    return k;
}
constexpr uint64_t kEmptyCell = ~0ULL;

__device__ __forceinline__ int find_seq(const SeqInfo* seqs, int B, int64_t i) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (seqs[mid].lo <= i) lo = mid; else hi = mid - 1;
    }
    return lo;
}

}  // namespace ssa

// The opaque handle of the C ABI is the plan itself.
struct ssa_plan_s : public ssa::Plan {};
