// C ABI of libssa.so (declared in include/ssa.h): argument validation, the plan object and its
// device buffers, the cached forward workspace, and dispatch to the kernels.
#include <algorithm>
#include <chrono>
#include <cstdio>
#include <cstdlib>
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "common.cuh"

namespace ssa {

std::atomic<int64_t> g_launches{0};

void trace_step(const char* what, cudaStream_t st) {
    static const bool on = [] {
        const char* e = getenv("SSA_TRACE");
        return e && e[0] == '1';
    }();
    if (!on) return;
    fprintf(stderr, "[ssa] %s: queued\n", what);
    fflush(stderr);
    auto t0 = std::chrono::steady_clock::now();
    cudaError_t e = cudaStreamSynchronize(st);
    double ms = std::chrono::duration<double, std::milli>(std::chrono::steady_clock::now() - t0).count();
    fprintf(stderr, "[ssa] %s: done %.3f ms (%s)\n", what, ms, cudaGetErrorString(e));
    fflush(stderr);
}

namespace {
std::mutex g_prof_mu;
bool g_prof_on = false;
struct ProfRec {
    const char* name;
    cudaEvent_t a, b;
};
std::vector<ProfRec> g_prof_pending;
std::vector<cudaEvent_t> g_prof_free;
struct ProfSum {
    std::string name;
    double ms = 0.0;
    int64_t launches = 0;
};
std::vector<ProfSum> g_prof_sums;

void prof_drain_locked() {
    for (auto& r : g_prof_pending) {
        float ms = 0.0f;
        cudaEventSynchronize(r.b);
        cudaEventElapsedTime(&ms, r.a, r.b);
        ProfSum* slot = nullptr;
        for (auto& x : g_prof_sums)
            if (x.name == r.name) slot = &x;
        if (!slot) {
            g_prof_sums.push_back(ProfSum{r.name, 0.0, 0});
            slot = &g_prof_sums.back();
        }
        slot->ms += ms;
        slot->launches += 1;
        g_prof_free.push_back(r.a);
        g_prof_free.push_back(r.b);
    }
    g_prof_pending.clear();
}
}  // namespace

bool profiling_on() { return g_prof_on; }

cudaEvent_t profile_event() {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (!g_prof_free.empty()) {
        cudaEvent_t e = g_prof_free.back();
        g_prof_free.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

void profile_record(const char* name, cudaEvent_t start, cudaEvent_t stop) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_pending.push_back(ProfRec{name, start, stop});
    if (g_prof_pending.size() > 4096) prof_drain_locked();
}

namespace {

// The default hook allocates stream-ordered from a memory pool owned by this library (one per
// device) whose release threshold keeps freed memory for reuse: a plan rebuilt every step then
// allocates from cached memory instead of mapping new pages at every synchronisation.
cudaMemPool_t library_pool() {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.handleTypes = cudaMemHandleTypeNone;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        uint64_t keep = ~0ull;
        cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        pools[dev] = pool;
    }
    return pools[dev];
}

void* default_alloc(size_t bytes, void* stream, void*) {
    void* p = nullptr;
    cudaMemPool_t pool = library_pool();
    const cudaError_t e = pool ? cudaMallocFromPoolAsync(&p, bytes, pool, (cudaStream_t)stream)
                               : cudaMallocAsync(&p, bytes, (cudaStream_t)stream);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return p;
}
void default_free(void* p, void* stream, void*) { cudaFreeAsync(p, (cudaStream_t)stream); }

std::mutex g_alloc_mu;
ssa_alloc_fn g_alloc = default_alloc;
ssa_free_fn g_free = default_free;
void* g_alloc_ctx = nullptr;

bool check_device(ssa_status_t* st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        *st = SSA_ERR_CUDA;
        return false;
    }
    int major = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (major != 10) {
        *st = SSA_ERR_UNSUPPORTED;
        return false;
    }
    return true;
}

size_t elem_size(ssa_dtype_t t) { return t == SSA_F32 ? 4 : 2; }

void free_host_pipe(Plan* p) {
    HostPipe& hp = p->hp;
    if (hp.s_in) cudaStreamSynchronize(hp.s_in);
    if (hp.s_out) cudaStreamSynchronize(hp.s_out);
    plan_free_all(p, hp.owned);
    for (cudaEvent_t e : {hp.e_in[0], hp.e_in[1], hp.e_comp[0], hp.e_comp[1], hp.e_out[0], hp.e_out[1],
                          hp.e_par, hp.e_start})
        if (e) cudaEventDestroy(e);
    if (hp.s_in) cudaStreamDestroy(hp.s_in);
    if (hp.s_out) cudaStreamDestroy(hp.s_out);
    hp = HostPipe();
}

void destroy(Plan* p) {
    ssa_plan_s* h = static_cast<ssa_plan_s*>(p);
    if (!p) return;
    plan_free_all(p, p->ws.owned);
    plan_free_all(p, p->ws_chunk.owned);
    free_host_pipe(p);
    destroy_blas(p);
    plan_free_all(p, p->owned);
    if (p->ws.h_q) cudaStreamSynchronize(p->stream);
    delete h;
}

ssa_status_t map_device_status(int32_t s) {
    if (!s) return SSA_OK;
    if (s & DEV_TIMEOUT) return SSA_ERR_DEVICE_TIMEOUT;
    if (s & DEV_COORD_RANGE) return SSA_ERR_COORD_RANGE;
    if (s & DEV_DUPLICATE) return SSA_ERR_DUPLICATE_COORD;
    if (s & DEV_TOO_LARGE) return SSA_ERR_UNSUPPORTED;
    return SSA_ERR_CUDA;
}

ssa_status_t make_plan(const int32_t* coords, const int64_t* cu, int32_t B, const int32_t* grids,
                       int32_t block, int32_t r, void* stream, ssa_plan_t* out) {
    if (!out) return SSA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!coords || !cu || !grids || B < 1 || B > 65535) return SSA_ERR_INVALID_ARG;
    if (block != kBlockEdge || r < 0 || r > kBlockEdge) return SSA_ERR_UNSUPPORTED;
    if (cu[0] != 0) return SSA_ERR_INVALID_ARG;
    for (int s = 0; s < B; ++s) {
        if (cu[s + 1] < cu[s]) return SSA_ERR_INVALID_ARG;
        for (int a = 0; a < 3; ++a)
            if (grids[3 * s + a] < 1 || grids[3 * s + a] > 65535) return SSA_ERR_INVALID_ARG;
    }
    const int64_t N = cu[B];
    if (N < 1 || N >= (int64_t)1 << 26) return SSA_ERR_INVALID_ARG;
    ssa_status_t st = SSA_OK;
    if (!check_device(&st)) return st;

    ssa_plan_s* p = new (std::nothrow) ssa_plan_s();
    if (!p) return SSA_ERR_ALLOC;
    {
        std::lock_guard<std::mutex> lk(g_alloc_mu);
        p->alloc = g_alloc;
        p->release = g_free;
        p->alloc_ctx = g_alloc_ctx;
    }
    cudaGetDevice(&p->device);
    p->stream = (cudaStream_t)stream;
    p->N = N;
    p->B = B;
    p->r = r;
    int64_t dense = 0;
    for (int s = 0; s < B; ++s) {
        SeqInfo q;
        q.lo = cu[s];
        q.hi = cu[s + 1];
        q.gx = grids[3 * s];
        q.gy = grids[3 * s + 1];
        q.gz = grids[3 * s + 2];
        q.gbx = (int32_t)cdiv(q.gx, kBlockEdge);
        q.gby = (int32_t)cdiv(q.gy, kBlockEdge);
        q.gbz = (int32_t)cdiv(q.gz, kBlockEdge);
        q.dense_base = dense;
        dense += (int64_t)q.gbx * q.gby * q.gbz;
        p->seqs.push_back(q);
    }
    p->G = dense;
    if (p->G >= ((int64_t)1 << 30)) {
        delete p;
        return SSA_ERR_UNSUPPORTED;
    }
    {
        ProfScope ps("plan", (cudaStream_t)stream);
        st = build_plan(p, coords, (cudaStream_t)stream);
    }
    if (st != SSA_OK) {
        cudaStreamSynchronize((cudaStream_t)stream);
        cudaGetLastError();
        destroy(p);
        return st;
    }
    *out = p;
    return SSA_OK;
}

// (Re)allocates the forward workspace for (H, D, dtype, k) if the cached one does not match.
ssa_status_t ensure_workspace(Plan* p, Workspace& w, int32_t H, int32_t D, ssa_dtype_t dt, int32_t k,
                              cudaStream_t st) {
    if (w.H == H && w.D == D && w.dtype == dt && w.k == k && w.kc) return SSA_OK;
    plan_free_all(p, w.owned);
    w = Workspace();
    const size_t es = elem_size(dt);
    const int64_t N = p->N, Mb = p->Mb;
    auto A = [&](size_t bytes) -> void* {
        void* ptr = p->alloc(std::max<size_t>(bytes, 16), st, p->alloc_ctx);
        if (ptr) w.owned.push_back(ptr);
        return ptr;
    };
    w.kc = A(es * H * Mb * D);
    w.vc = A(es * H * Mb * D);
    w.sel = (int32_t*)A(sizeof(int32_t) * N * H * k);
    if (!w.kc || !w.vc || !w.sel) return SSA_ERR_ALLOC;
    if (dt != SSA_F32) {
        w.Mb8 = round_up(Mb, 8);
        w.ks = A(es * H * p->Nks * D);
        w.vs = A(es * H * p->Nks * D);
        w.kcg = A(es * H * w.Mb8 * D);
        w.vcg = A(es * H * w.Mb8 * D);
        w.base = (float*)A(sizeof(float) * p->n_qtiles * kQTile * H * D);
        if (!w.ks || !w.vs || !w.kcg || !w.vcg || !w.base) return SSA_ERR_ALLOC;
        // padding rows of the block-ordered copies stay zero for the life of the workspace
        if (cudaMemsetAsync(w.ks, 0, es * H * p->Nks * D, st) ||
            cudaMemsetAsync(w.vs, 0, es * H * p->Nks * D, st) ||
            cudaMemsetAsync(w.kcg, 0, es * H * w.Mb8 * D, st) ||
            cudaMemsetAsync(w.vcg, 0, es * H * w.Mb8 * D, st))
            return SSA_ERR_CUDA;
    }
    w.H = H;
    w.D = D;
    w.dtype = dt;
    w.k = k;
    return SSA_OK;
}

ssa_status_t check_forward_args(Plan* p, const void* q, const void* k, const void* v,
                                const float* gates, const float* wc, int32_t H, int32_t D,
                                ssa_dtype_t dt, int32_t topk, const void* out) {
    if (!p || !q || !k || !v || !gates || !wc || !out) return SSA_ERR_INVALID_ARG;
    if (dt != SSA_F32 && dt != SSA_BF16 && dt != SSA_F16) return SSA_ERR_INVALID_ARG;
    if (H < 1 || topk < 1) return SSA_ERR_INVALID_ARG;
    if (topk > kMaxTopk) return SSA_ERR_UNSUPPORTED;
    if (D != 32 && D != 64 && D != 96 && D != 128) return SSA_ERR_UNSUPPORTED;
    const int64_t hd = (int64_t)H * D;
    if (hd > (dt == SSA_F32 ? 8192 : 16384)) return SSA_ERR_UNSUPPORTED;
    if (p->N * H >= ((int64_t)1 << 31) / std::max(topk, 1)) return SSA_ERR_UNSUPPORTED;
    return SSA_OK;
}

// What a forward call computes beyond the plain method (everything off by default).
struct Options {
    Prologue pro;
    const float* conv_w = nullptr;   // [27, D, D]: compression by sparse 3D convolution
    const float* gate_w = nullptr;   // [D, 3] and [3]: gates predicted from the queries
    const float* gate_b = nullptr;
    bool share = false;              // one selection per 4x4x4 sub-block (16-bit types)
};

// A workspace buffer of `bytes` allocated on first use (kept with the workspace).
template <typename P>
ssa_status_t ensure_buffer(Plan* p, Workspace& w, P*& buf, size_t bytes, cudaStream_t st) {
    if (buf) return SSA_OK;
    buf = (P*)p->alloc(std::max<size_t>(bytes, 16), st, p->alloc_ctx);
    if (!buf) return SSA_ERR_ALLOC;
    w.owned.push_back(buf);
    return SSA_OK;
}

ssa_status_t run_forward(Plan* p, const void* q, const void* k, const void* v, const float* gates,
                         const float* wc, int32_t H, int32_t D, ssa_dtype_t dt, int32_t topk,
                         void* out, int32_t* sel_out, cudaStream_t st,
                         const BranchOut& bo = BranchOut(), const Options& opt = Options(),
                         Workspace* wsp = nullptr) {
    Workspace& w = wsp ? *wsp : p->ws;
    ssa_status_t rc = ensure_workspace(p, w, H, D, dt, topk, st);
    if (rc != SSA_OK) return rc;
    const Prologue& pro = opt.pro;
    if (pro.on() && dt == SSA_F32) {
        // fp32 path: the prologue is a pass of its own into workspace copies of q and k
        const size_t bytes = sizeof(float) * (size_t)p->N * H * D;
        if ((rc = ensure_buffer(p, w, w.qp, bytes, st)) != SSA_OK) return rc;
        if ((rc = ensure_buffer(p, w, w.kp, bytes, st)) != SSA_OK) return rc;
        {
            ProfScope ps("prologue", st);
            launch_qk_prologue_f32(p, (const float*)q, pro.q_gamma, pro, H, D, w.qp, st);
            launch_qk_prologue_f32(p, (const float*)k, pro.k_gamma, pro, H, D, w.kp, st);
        }
        q = w.qp;
        k = w.kp;
    }
    const Prologue fused = dt == SSA_F32 ? Prologue() : pro;   // 16-bit: inside pool and forward
    float* means = nullptr;
    if (opt.conv_w) {
        if ((rc = ensure_block_neighbours(p, st)) != SSA_OK) return rc;
        if ((rc = ensure_buffer(p, w, w.means, sizeof(float) * 2 * (size_t)H * p->Mb * D, st)) != SSA_OK)
            return rc;
        means = w.means;
    }
    {
        ProfScope ps("pool", st);
        launch_pool(p, w, k, v, wc, fused, means, st);
    }
    if (opt.conv_w) {
        ProfScope ps("conv", st);
        launch_conv_compress(p, w, means, opt.conv_w, st);
    }
    trace_step("pool", st);
    if (opt.gate_w) {
        if ((rc = ensure_buffer(p, w, w.gates, sizeof(float) * 3 * (size_t)p->N * H, st)) != SSA_OK) return rc;
        gates = w.gates;
        if (dt == SSA_F32) launch_gates_f32(p, (const float*)q, opt.gate_w, opt.gate_b, H, D, w.gates, st);
    }
    if (dt == SSA_F32) {
        // the CUDA-core path walks the per-token neighbour lists
        if ((rc = ensure_neighbours(p, st)) != SSA_OK) return rc;
        launch_forward_simt(p, w, q, k, v, gates, out, bo, st);
    } else {
        if (opt.share) {
            if ((rc = ensure_subblock_tiles(p, st)) != SSA_OK) return rc;
            rc = launch_select_shared(p, w, q, fused, opt.gate_w, opt.gate_b, opt.gate_w ? w.gates : nullptr, st);
        } else {
            rc = launch_select_tc(p, w, q, fused, opt.gate_w, opt.gate_b, opt.gate_w ? w.gates : nullptr, st);
        }
        if (rc != SSA_OK) return rc;
        trace_step("select", st);
        if ((rc = launch_forward_tc(p, w, q, gates, out, bo, fused, st)) != SSA_OK) return rc;
    }
    trace_step("forward", st);
    if (sel_out) launch_export_sel(p, w, sel_out, st);
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

// Gates of heads [h0, h0 + hc) of [N, H, 3] into [N, hc, 3].
__global__ void k_gather_gates(const float* __restrict__ in, int64_t N, int H, int h0, int hc,
                               float* __restrict__ out) {
    const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= N * hc * 3) return;
    const int64_t n = e / (hc * 3), r = e % (hc * 3);
    out[e] = in[(n * H + h0) * 3 + r];
}

// Heads per chunk of the host-buffer path: the smallest divisor of H whose rows of one token are
// at least 256 bytes (efficient strided copies); H itself (no chunking) if there is none below H.
int32_t host_chunk_heads(int32_t H, int32_t D, ssa_dtype_t dt) {
    const size_t es = elem_size(dt);
    for (int32_t d = 1; d < H; ++d)
        if (H % d == 0 && (size_t)d * D * es >= 256) return d;
    return H;
}

ssa_status_t ensure_host_pipe(Plan* p, int32_t H, int32_t D, ssa_dtype_t dt, int32_t hc, cudaStream_t st) {
    HostPipe& hp = p->hp;
    if (hp.hc == hc && hp.H == H && hp.D == D && hp.dtype == dt) return SSA_OK;
    free_host_pipe(p);
    if (cudaStreamCreateWithFlags(&hp.s_in, cudaStreamNonBlocking) ||
        cudaStreamCreateWithFlags(&hp.s_out, cudaStreamNonBlocking))
        return SSA_ERR_CUDA;
    for (cudaEvent_t* e : {&hp.e_in[0], &hp.e_in[1], &hp.e_comp[0], &hp.e_comp[1], &hp.e_out[0], &hp.e_out[1],
                           &hp.e_par, &hp.e_start})
        if (cudaEventCreateWithFlags(e, cudaEventDisableTiming)) return SSA_ERR_CUDA;
    const size_t cb = elem_size(dt) * (size_t)p->N * hc * D;
    auto A = [&](size_t bytes) -> void* {
        void* ptr = p->alloc(std::max<size_t>(bytes, 16), st, p->alloc_ctx);
        if (ptr) hp.owned.push_back(ptr);
        return ptr;
    };
    for (int s = 0; s < 2; ++s) {
        hp.q[s] = A(cb);
        hp.k[s] = A(cb);
        hp.v[s] = A(cb);
        hp.o[s] = A(cb);
        hp.g[s] = (float*)A(sizeof(float) * 3 * (size_t)p->N * hc);
        if (!hp.q[s] || !hp.k[s] || !hp.v[s] || !hp.o[s] || !hp.g[s]) return SSA_ERR_ALLOC;
    }
    hp.gates = (float*)A(sizeof(float) * 3 * (size_t)p->N * H);
    hp.wc = (float*)A(sizeof(float) * (size_t)D * D);
    if (!hp.gates || !hp.wc) return SSA_ERR_ALLOC;
    // the buffers come from the caller's stream: the side streams wait for their allocation
    if (cudaEventRecord(hp.e_start, st) || cudaStreamWaitEvent(hp.s_in, hp.e_start, 0) ||
        cudaStreamWaitEvent(hp.s_out, hp.e_start, 0))
        return SSA_ERR_CUDA;
    hp.hc = hc;
    hp.H = H;
    hp.D = D;
    hp.dtype = dt;
    return SSA_OK;
}

// The host-buffer forward, heads in chunks of hc: chunk c's inputs are copied in on s_in (strided
// rows of the [N, H, D] host tensors) while chunk c - 1 runs on the caller's stream and chunk
// c - 2's output is copied out on s_out. Two slots of buffers; events order their reuse.
ssa_status_t forward_host_chunked(Plan* p, const void* q, const void* k, const void* v, const float* gates,
                                  const float* wc, int32_t H, int32_t D, ssa_dtype_t dt, int32_t topk,
                                  void* out, int32_t hc, cudaStream_t st) {
    ssa_status_t rc = ensure_host_pipe(p, H, D, dt, hc, st);
    if (rc != SSA_OK) return rc;
    HostPipe& hp = p->hp;
    const size_t es = elem_size(dt), row = es * (size_t)H * D, crow = es * (size_t)hc * D;
    const int64_t N = p->N;
    const int nch = H / hc;
    const auto H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;
    // work the caller queued before this call (a plan rebuild) comes first on every stream
    if (cudaEventRecord(hp.e_start, st) || cudaStreamWaitEvent(hp.s_in, hp.e_start, 0) ||
        cudaStreamWaitEvent(hp.s_out, hp.e_start, 0))
        return SSA_ERR_CUDA;
    if (cudaMemcpyAsync(hp.gates, gates, sizeof(float) * 3 * (size_t)N * H, H2D, hp.s_in) ||
        cudaMemcpyAsync(hp.wc, wc, sizeof(float) * (size_t)D * D, H2D, hp.s_in) ||
        cudaEventRecord(hp.e_par, hp.s_in))
        return SSA_ERR_CUDA;
    for (int c = 0; c < nch; ++c) {
        const int s = c & 1;
        const size_t h0 = (size_t)c * hc * D * es;
        // copies in: the slot's previous chunk must be done with its inputs
        if (c >= 2 && cudaStreamWaitEvent(hp.s_in, hp.e_comp[s], 0)) return SSA_ERR_CUDA;
        if (cudaMemcpy2DAsync(hp.q[s], crow, (const uint8_t*)q + h0, row, crow, (size_t)N, H2D, hp.s_in) ||
            cudaMemcpy2DAsync(hp.k[s], crow, (const uint8_t*)k + h0, row, crow, (size_t)N, H2D, hp.s_in) ||
            cudaMemcpy2DAsync(hp.v[s], crow, (const uint8_t*)v + h0, row, crow, (size_t)N, H2D, hp.s_in) ||
            cudaEventRecord(hp.e_in[s], hp.s_in))
            return SSA_ERR_CUDA;
        // the forward of the chunk: its inputs are in, the slot's previous output is out
        if (cudaStreamWaitEvent(st, hp.e_in[s], 0) || (c == 0 && cudaStreamWaitEvent(st, hp.e_par, 0)) ||
            (c >= 2 && cudaStreamWaitEvent(st, hp.e_out[s], 0)))
            return SSA_ERR_CUDA;
        const int64_t ng = N * hc * 3;
        if (ng > 0) {
            k_gather_gates<<<(unsigned)cdiv(ng, 256), 256, 0, st>>>(hp.gates, N, H, c * hc, hc, hp.g[s]);
            note_launch();
        }
        rc = run_forward(p, hp.q[s], hp.k[s], hp.v[s], hp.g[s], hp.wc, hc, D, dt, topk, hp.o[s], nullptr, st,
                         BranchOut(), Options(), &p->ws_chunk);
        if (rc != SSA_OK) return rc;
        if (cudaEventRecord(hp.e_comp[s], st)) return SSA_ERR_CUDA;
        // copies out
        if (cudaStreamWaitEvent(hp.s_out, hp.e_comp[s], 0) ||
            cudaMemcpy2DAsync((uint8_t*)out + h0, row, hp.o[s], crow, crow, (size_t)N, D2H, hp.s_out) ||
            cudaEventRecord(hp.e_out[s], hp.s_out))
            return SSA_ERR_CUDA;
    }
    // the caller's stream completes after the last copies out
    for (int s = 0; s < 2 && s < nch; ++s)
        if (cudaStreamWaitEvent(st, hp.e_out[s], 0)) return SSA_ERR_CUDA;
    return SSA_OK;
}

}  // namespace

void* plan_alloc(Plan* p, size_t bytes) {
    void* ptr = p->alloc(std::max<size_t>(bytes, 16), p->stream, p->alloc_ctx);
    if (ptr) p->owned.push_back(ptr);
    return ptr;
}

void plan_free_all(Plan* p, std::vector<void*>& list) {
    for (void* ptr : list) p->release(ptr, p->stream, p->alloc_ctx);
    list.clear();
}

}  // namespace ssa

using namespace ssa;

extern "C" {

ssa_status_t ssa_set_allocator(ssa_alloc_fn alloc, ssa_free_fn release, void* ctx) {
    if ((alloc == nullptr) != (release == nullptr)) return SSA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_alloc_mu);
    g_alloc = alloc ? alloc : default_alloc;
    g_free = release ? release : default_free;
    g_alloc_ctx = alloc ? ctx : nullptr;
    return SSA_OK;
}

ssa_status_t ssa_plan(const int32_t* coords, int64_t n, const int32_t grid[3], int32_t block,
                      int32_t r, void* stream, ssa_plan_t* out) {
    if (!grid || n < 1) return SSA_ERR_INVALID_ARG;
    int64_t cu[2] = {0, n};
    return make_plan(coords, cu, 1, grid, block, r, stream, out);
}

ssa_status_t ssa_plan_varlen(const int32_t* coords, const int64_t* cu_seqlens, int32_t batch,
                             const int32_t* grids, int32_t block, int32_t r, void* stream,
                             ssa_plan_t* out) {
    return make_plan(coords, cu_seqlens, batch, grids, block, r, stream, out);
}

ssa_status_t ssa_plan_rebuild(ssa_plan_t p, const int32_t* coords, void* stream) {
    if (!p || !coords) return SSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t old_mb = p->Mb, old_nks = p->Nks;
    plan_free_all(p, p->owned);
    p->stream = st;
    ssa_status_t rc;
    {
        ProfScope ps("plan", st);
        rc = build_plan(p, coords, st);
    }
    if (rc != SSA_OK) {
        cudaStreamSynchronize(st);
        cudaGetLastError();
        plan_free_all(p, p->owned);
        plan_free_all(p, p->ws.owned);
        p->ws = Workspace();
        plan_free_all(p, p->ws_chunk.owned);
        p->ws_chunk = Workspace();
        return rc;
    }
    if (p->Mb != old_mb || p->Nks != old_nks) {
        plan_free_all(p, p->ws.owned);
        p->ws = Workspace();
        plan_free_all(p, p->ws_chunk.owned);
        p->ws_chunk = Workspace();
    }
    return SSA_OK;
}

ssa_status_t ssa_plan_info(ssa_plan_t plan, int64_t* n, int64_t* num_blocks, int64_t* nnz,
                           int32_t* batch) {
    if (!plan) return SSA_ERR_INVALID_ARG;
    if (n) *n = plan->N;
    if (num_blocks) *num_blocks = plan->Mb;
    if (nnz) {
        const ssa_status_t rc = ensure_neighbour_counts(plan, plan->stream);
        if (rc != SSA_OK) return rc;
        *nnz = plan->nnz;
    }
    if (batch) *batch = plan->B;
    return SSA_OK;
}

ssa_status_t ssa_plan_export(ssa_plan_t p, int32_t* perm, int32_t* tok_blk, int32_t* blk_off,
                             int32_t* blk_coord, int32_t* blk_seq, int64_t* nbr_off,
                             int32_t* nbr_idx, void* stream) {
    if (!p) return SSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    const auto D2D = cudaMemcpyDeviceToDevice;
    if (nbr_idx || nbr_off) {
        const ssa_status_t rc = nbr_idx ? ensure_neighbours(p, st) : ensure_neighbour_counts(p, st);
        if (rc != SSA_OK) return rc;
    }
    cudaError_t e = cudaSuccess;
    if (perm && !e) e = cudaMemcpyAsync(perm, p->perm, sizeof(int32_t) * p->N, D2D, st);
    if (tok_blk && !e) e = cudaMemcpyAsync(tok_blk, p->tok_blk, sizeof(int32_t) * p->N, D2D, st);
    if (blk_off && !e) e = cudaMemcpyAsync(blk_off, p->blk_off, sizeof(int32_t) * (p->Mb + 1), D2D, st);
    if (blk_coord && !e) e = cudaMemcpyAsync(blk_coord, p->blk_coord, sizeof(int32_t) * 3 * p->Mb, D2D, st);
    if (blk_seq && !e) e = cudaMemcpyAsync(blk_seq, p->blk_seq, sizeof(int32_t) * p->Mb, D2D, st);
    if (nbr_idx && !e && p->nnz) e = cudaMemcpyAsync(nbr_idx, p->nbr_idx, sizeof(int32_t) * p->nnz, D2D, st);
    if (nbr_off && !e) {
        std::vector<int32_t> h32(p->N + 1);
        std::vector<int64_t> h64(p->N + 1);
        e = cudaMemcpyAsync(h32.data(), p->nbr_off32, sizeof(int32_t) * (p->N + 1), cudaMemcpyDeviceToHost, st);
        if (!e) e = cudaStreamSynchronize(st);
        for (int64_t i = 0; i <= p->N && !e; ++i) h64[i] = h32[i];
        if (!e) e = cudaMemcpyAsync(nbr_off, h64.data(), sizeof(int64_t) * (p->N + 1), cudaMemcpyHostToDevice, st);
    }
    if (!e) e = cudaStreamSynchronize(st);
    return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

ssa_status_t ssa_forward(ssa_plan_t p, const void* q, const void* k, const void* v,
                         const float* gates, const float* wc, int32_t heads, int32_t head_dim,
                         ssa_dtype_t dtype, int32_t topk, void* out, void* stream) {
    ssa_status_t rc = check_forward_args(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out);
    if (rc != SSA_OK) return rc;
    return run_forward(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out, nullptr,
                       (cudaStream_t)stream);
}

ssa_status_t ssa_forward_debug(ssa_plan_t p, const void* q, const void* k, const void* v,
                               const float* gates, const float* wc, int32_t heads,
                               int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* out,
                               int32_t* sel_out, float* o_cmp, float* o_sel, float* o_win,
                               void* stream) {
    ssa_status_t rc = check_forward_args(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out);
    if (rc != SSA_OK) return rc;
    BranchOut bo;
    bo.o[0] = o_cmp;
    bo.o[1] = o_sel;
    bo.o[2] = o_win;
    return run_forward(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out, sel_out,
                       (cudaStream_t)stream, bo);
}

ssa_status_t ssa_forward_prologue(ssa_plan_t p, const void* q, const void* k, const void* v,
                                  const float* gates, const float* wc, const float* q_gamma,
                                  const float* k_gamma, float rope_theta, float eps, int32_t heads,
                                  int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* out,
                                  int32_t* sel_out, void* stream) {
    ssa_status_t rc = check_forward_args(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out);
    if (rc != SSA_OK) return rc;
    if (!q_gamma || !k_gamma || !(rope_theta > 1.0f) || !(eps >= 0.0f)) return SSA_ERR_INVALID_ARG;
    Options opt;
    opt.pro.q_gamma = q_gamma;
    opt.pro.k_gamma = k_gamma;
    opt.pro.theta = rope_theta;
    opt.pro.eps = eps;
    return run_forward(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out, sel_out,
                       (cudaStream_t)stream, BranchOut(), opt);
}

ssa_status_t ssa_forward_ex(ssa_plan_t p, const void* q, const void* k, const void* v,
                            const float* gates, const float* wc, int32_t heads, int32_t head_dim,
                            ssa_dtype_t dtype, int32_t topk, const ssa_options_t* options, void* out,
                            int32_t* sel_out, void* stream) {
    Options opt;
    if (options) {
        const ssa_options_t& o = *options;
        if ((o.q_gamma == nullptr) != (o.k_gamma == nullptr)) return SSA_ERR_INVALID_ARG;
        if (o.q_gamma && (!(o.rope_theta > 1.0f) || !(o.rms_eps >= 0.0f))) return SSA_ERR_INVALID_ARG;
        if ((o.gate_w == nullptr) != (o.gate_b == nullptr)) return SSA_ERR_INVALID_ARG;
        opt.pro.q_gamma = o.q_gamma;
        opt.pro.k_gamma = o.k_gamma;
        opt.pro.theta = o.rope_theta;
        opt.pro.eps = o.rms_eps;
        opt.conv_w = o.conv_w;
        opt.gate_w = o.gate_w;
        opt.gate_b = o.gate_b;
        if (o.select_share != 0 && o.select_share != 1) return SSA_ERR_INVALID_ARG;
        opt.share = o.select_share == 1;
        if (opt.share && dtype == SSA_F32) return SSA_ERR_UNSUPPORTED;
    }
    // the gates input is not read when they are predicted, nor wc with a convolution compression
    static const float kUnused = 0.0f;
    ssa_status_t rc = check_forward_args(p, q, k, v, opt.gate_w ? &kUnused : gates, opt.conv_w ? &kUnused : wc,
                                         heads, head_dim, dtype, topk, out);
    if (rc != SSA_OK) return rc;
    return run_forward(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out, sel_out,
                       (cudaStream_t)stream, BranchOut(), opt);
}

ssa_status_t ssa_forward_host(ssa_plan_t p, const void* q, const void* k, const void* v,
                              const float* gates, const float* wc, int32_t heads,
                              int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* out,
                              void* stream) {
    ssa_status_t rc = check_forward_args(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out);
    if (rc != SSA_OK) return rc;
    cudaStream_t st = (cudaStream_t)stream;
    const int32_t hc = host_chunk_heads(heads, head_dim, dtype);
    if (hc < heads) {
        if ((rc = forward_host_chunked(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, out, hc, st)) != SSA_OK)
            return rc;
    } else {
        Workspace& w = p->ws;
        const size_t tb = elem_size(dtype) * (size_t)p->N * heads * head_dim;
        const size_t gb = sizeof(float) * (size_t)p->N * heads * 3;
        const size_t wb = sizeof(float) * (size_t)head_dim * head_dim;
        rc = ensure_workspace(p, w, heads, head_dim, dtype, topk, st);
        if (rc != SSA_OK) return rc;
        if (!w.h_q) {
            void* bufs[6];
            const size_t sizes[6] = {tb, tb, tb, tb, gb, wb};
            for (int i = 0; i < 6; ++i) {
                bufs[i] = p->alloc(sizes[i], st, p->alloc_ctx);
                if (!bufs[i]) return SSA_ERR_ALLOC;
                w.owned.push_back(bufs[i]);
            }
            w.h_q = bufs[0];
            w.h_k = bufs[1];
            w.h_v = bufs[2];
            w.h_out = bufs[3];
            w.h_gates = (float*)bufs[4];
            w.h_wc = (float*)bufs[5];
        }
        const auto H2D = cudaMemcpyHostToDevice;
        if (cudaMemcpyAsync(w.h_q, q, tb, H2D, st) || cudaMemcpyAsync(w.h_k, k, tb, H2D, st) ||
            cudaMemcpyAsync(w.h_v, v, tb, H2D, st) || cudaMemcpyAsync(w.h_gates, gates, gb, H2D, st) ||
            cudaMemcpyAsync(w.h_wc, wc, wb, H2D, st))
            return SSA_ERR_CUDA;
        rc = run_forward(p, w.h_q, w.h_k, w.h_v, w.h_gates, w.h_wc, heads, head_dim, dtype, topk,
                         w.h_out, nullptr, st);
        if (rc != SSA_OK) return rc;
        if (cudaMemcpyAsync(out, w.h_out, tb, cudaMemcpyDeviceToHost, st)) return SSA_ERR_CUDA;
    }
    if (cudaStreamSynchronize(st)) return SSA_ERR_CUDA;
    int32_t s = 0;
    if (cudaMemcpy(&s, p->d_status, sizeof(int32_t), cudaMemcpyDeviceToHost)) return SSA_ERR_CUDA;
    return map_device_status(s);
}

ssa_status_t ssa_backward(ssa_plan_t p, const void* q, const void* k, const void* v,
                          const float* gates, const float* wc, const void* dout, int32_t heads,
                          int32_t head_dim, ssa_dtype_t dtype, int32_t topk, void* dq, void* dk,
                          void* dv, void* stream) {
    ssa_status_t rc = check_forward_args(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, dq);
    if (rc != SSA_OK) return rc;
    if (!dout || !dk || !dv) return SSA_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    rc = ensure_workspace(p, p->ws, heads, head_dim, dtype, topk, st);
    if (rc != SSA_OK) return rc;
    // the selection is the forward's: run the forward path to produce it (output goes to dq,
    // which the backward overwrites)
    rc = run_forward(p, q, k, v, gates, wc, heads, head_dim, dtype, topk, dq, nullptr, st);
    if (rc != SSA_OK) return rc;
    if ((rc = ensure_neighbours(p, st)) != SSA_OK) return rc;
    return launch_backward(p, p->ws, q, k, v, gates, wc, dout, dq, dk, dv, st);
}

ssa_status_t ssa_last_device_status(ssa_plan_t p, void* stream) {
    if (!p) return SSA_ERR_INVALID_ARG;
    int32_t s = 0;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaStreamSynchronize(st) ||
        cudaMemcpyAsync(&s, p->d_status, sizeof(int32_t), cudaMemcpyDeviceToHost, st) ||
        cudaMemsetAsync(p->d_status, 0, sizeof(int32_t), st) || cudaStreamSynchronize(st))
        return SSA_ERR_CUDA;
    return map_device_status(s);
}

ssa_status_t ssa_debug_wait_timeout(ssa_plan_t p, int64_t max_cycles, void* stream) {
    if (!p || max_cycles < 1) return SSA_ERR_INVALID_ARG;
    return launch_wait_timeout(p, max_cycles, (cudaStream_t)stream);
}

ssa_status_t ssa_plan_destroy(ssa_plan_t p) {
    if (!p) return SSA_ERR_INVALID_ARG;
    destroy(p);
    return SSA_OK;
}

const char* ssa_status_string(ssa_status_t s) {
    switch (s) {
    case SSA_OK: return "ok";
    case SSA_ERR_INVALID_ARG: return "invalid argument";
    case SSA_ERR_COORD_RANGE: return "coordinate outside the grid";
    case SSA_ERR_DUPLICATE_COORD: return "duplicate coordinate";
    case SSA_ERR_ALLOC: return "device allocation failed";
    case SSA_ERR_CUDA: return "CUDA error";
    case SSA_ERR_UNSUPPORTED: return "unsupported size or device";
    case SSA_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

int64_t ssa_launch_count(void) { return g_launches.load(); }

ssa_status_t ssa_profile_enable(int32_t on) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = on != 0;
    return SSA_OK;
}

ssa_status_t ssa_profile_reset(void) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    prof_drain_locked();
    g_prof_sums.clear();
    return SSA_OK;
}

int32_t ssa_profile_read(int32_t max_entries, char* names, double* total_ms, int64_t* launches) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    prof_drain_locked();
    int32_t n = 0;
    for (auto& x : g_prof_sums) {
        if (n >= max_entries) break;
        if (names) {
            std::strncpy(names + 64 * n, x.name.c_str(), 63);
            names[64 * n + 63] = 0;
        }
        if (total_ms) total_ms[n] = x.ms;
        if (launches) launches[n] = x.launches;
        ++n;
    }
    return n;
}

}  // extern "C"
