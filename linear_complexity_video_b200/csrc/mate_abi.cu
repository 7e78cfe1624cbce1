// C ABI of the MATE token-mix library: argument checks, workspace layout and
// dispatch to the kernels. Declarations and contracts live in include/mate.h.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "../../include/mate.h"
#include "common.cuh"
#include "devctx.h"
#include "kernels.h"

namespace mate {

// Device-side error word: kernels with bounded waits or device checks set it;
// mate_last_error() reads and clears it.
__device__ int g_error_word = 0;

namespace {
std::atomic<uint64_t> g_launches{0};
mate_phase_hook g_hook = nullptr;
void *g_hook_user = nullptr;
}  // namespace

// Device address of g_error_word in the current device's context, looked up once
// per device and again after that device's context has been re-created.
int *error_word_ptr()
{
    static std::mutex mu;
    static int *addr[64] = {};
    static unsigned long long ctx_of[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || ctx != ctx_of[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_error_word) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<int *>(p);
        ctx_of[dev] = ctx;
    }
    return addr[dev];
}

void phase_mark(int phase, int is_end, cudaStream_t s)
{
    if (g_hook) g_hook(phase, is_end, static_cast<void *>(s), g_hook_user);
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

constexpr int kMaxChunk = 1024;        // longest chunk the state kernels take
constexpr int kMaxGenericChunk = 256;  // longest chunk of the CUDA-core output kernel
constexpr size_t kAlign = 256;
constexpr size_t kMaxSmem = 227 * 1024;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

bool supported_head(int v) { return v == 16 || v == 32 || v == 64; }

// Fill the shape part of SsdArgs and check it; returns MATE_OK or an error.
int ssd_shape(int T, int H, int W, const int *pool, const mate_ssd_dims *d, int scan_mode, SsdArgs &a)
{
    if (!d) return MATE_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || W <= 0 || d->batch <= 0 || d->nheads <= 0 || d->ngroups <= 0 || d->chunk <= 0)
        return MATE_ERR_INVALID_ARG;
    const int64_t N = (int64_t)T * H * W;
    if (N >= ((int64_t)1 << 31) || N * d->batch >= ((int64_t)1 << 40)) return MATE_ERR_INVALID_ARG;
    if (d->nheads % d->ngroups) return MATE_ERR_INVALID_ARG;
    if (scan_mode < 0 || scan_mode > MATE_SCAN_ZZ) return MATE_ERR_INVALID_ARG;
    const int dirs = d->directions == 0 ? MATE_DIR_BI : d->directions;
    if (dirs < 1 || dirs > 3) return MATE_ERR_INVALID_ARG;
    if (d->dtype != MATE_F32 && d->dtype != MATE_BF16) return MATE_ERR_UNSUPPORTED;
    if (!supported_head(d->headdim) || !supported_head(d->dstate)) return MATE_ERR_UNSUPPORTED;
    if (d->chunk > kMaxChunk) return MATE_ERR_UNSUPPORTED;
    memset(&a, 0, sizeof(a));
    a.batch = d->batch;
    a.T = T;
    a.H = H;
    a.W = W;
    a.N = (int)N;
    a.nh = d->nheads;
    a.P = d->headdim;
    a.Ns = d->dstate;
    a.G = d->ngroups;
    a.Q = d->chunk;
    a.nchunks = (int)((N + d->chunk - 1) / d->chunk);
    a.mode = scan_mode;
    a.dirs = dirs;
    a.bf16 = d->dtype == MATE_BF16;
    a.dT = make_fastdiv(T);
    a.dH = make_fastdiv(H);
    a.dW = make_fastdiv(W);
    a.dHW = make_fastdiv((uint32_t)(H * W));
    a.dpt = a.dph = a.dpw = make_fastdiv(1);
    const bool review = pool && (pool[0] || pool[1] || pool[2]);
    if (review) {
        if (pool[0] <= 0 || pool[1] <= 0 || pool[2] <= 0) return MATE_ERR_INVALID_ARG;
        if (T % pool[0] || H % pool[1] || W % pool[2]) return MATE_ERR_INVALID_ARG;
        a.review = 1;
        a.pt = pool[0];
        a.ph = pool[1];
        a.pw = pool[2];
        a.Tp = T / pool[0];
        a.Hp = H / pool[1];
        a.Wp = W / pool[2];
        a.Np = a.Tp * a.Hp * a.Wp;
        a.dpt = make_fastdiv(a.pt);
        a.dph = make_fastdiv(a.ph);
        a.dpw = make_fastdiv(a.pw);
        // split each pooling box so that the pooling grid covers the GPU a few times over
        const int64_t box = (int64_t)a.pt * a.ph * a.pw;
        const int64_t blocks = (int64_t)a.Np * a.batch * ((a.nh * a.P + a.nh + a.G * a.Ns) / 8 / 256 + 1);
        int64_t splits = (1184 + blocks - 1) / blocks;
        if (splits > 8) splits = 8;
        if (splits > box) splits = box;
        if (splits < 1) splits = 1;
        a.pool_splits = (int)splits;
    }
    return MATE_OK;
}

// Which kernels run a bi-SSD call: bf16 storage runs on the tensor-core kernels
// (1) and fp32 storage on the CUDA-core kernels (0); -1 when the kernels of that
// storage type cannot take the dims. There is no fallback from one to the other.
int ssd_path(const SsdArgs &a)
{
    if (a.bf16) return ssd_tc_supported(a) ? 1 : -1;
    const size_t smem = ((size_t)a.Q * (a.P + a.Ns) + 2 * a.P * a.Ns + 3 * (size_t)a.Q) * sizeof(float);
    if (a.Q > kMaxGenericChunk || smem > kMaxSmem) return -1;
    return 0;
}

void carve(SsdArgs &a, void *ws)
{
    const SsdWorkspace l = ssd_workspace_layout(a);
    char *base = static_cast<char *>(ws);
    a.states_f = reinterpret_cast<float *>(base + l.states_f);
    a.states_b = reinterpret_cast<float *>(base + l.states_b);
    a.alpha = reinterpret_cast<float *>(base + l.alpha);
    a.h_init = a.review ? reinterpret_cast<float *>(base + l.h_init) : nullptr;
    a.pooled = a.review ? reinterpret_cast<float *>(base + l.pooled) : nullptr;
    a.dt_scan = a.bf16 ? reinterpret_cast<float *>(base + l.dt_scan) : nullptr;
}

int attn_shape(int T, int H, int W, int Tw, int Sw, const int *shift, const mate_attn_dims *d, TesaArgs &a)
{
    if (!d || !shift) return MATE_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || W <= 0 || Tw <= 0 || Sw <= 0 || d->batch <= 0 || d->nheads <= 0)
        return MATE_ERR_INVALID_ARG;
    const int64_t N = (int64_t)T * H * W;
    if (N >= ((int64_t)1 << 31)) return MATE_ERR_INVALID_ARG;
    if (shift[0] < 0 || shift[0] >= Tw || shift[1] < 0 || shift[1] >= Sw || shift[2] < 0 || shift[2] >= Sw)
        return MATE_ERR_INVALID_ARG;
    if (d->dtype != MATE_F32 && d->dtype != MATE_BF16) return MATE_ERR_UNSUPPORTED;
    memset(&a, 0, sizeof(a));
    a.batch = d->batch;
    a.T = T;
    a.H = H;
    a.W = W;
    a.N = (int)N;
    a.nh = d->nheads;
    a.d = d->headdim;
    a.Tw = Tw;
    a.Sw = Sw;
    a.st = shift[0];
    a.sh = shift[1];
    a.sw = shift[2];
    a.offt = win_offset(Tw, shift[0]);
    a.offh = win_offset(Sw, shift[1]);
    a.offw = win_offset(Sw, shift[2]);
    a.nwt = (T + a.offt + Tw - 1) / Tw;
    a.nwh = (H + a.offh + Sw - 1) / Sw;
    a.nww = (W + a.offw + Sw - 1) / Sw;
    a.bf16 = d->dtype == MATE_BF16;
    return MATE_OK;
}

}  // namespace

SsdWorkspace ssd_workspace_layout(const SsdArgs &a)
{
    SsdWorkspace l;
    const size_t nstate = (size_t)a.batch * a.nh * a.nchunks * a.P * a.Ns;
    // chunk states: bf16 on the tensor-core path (bf16 storage), fp32 on the CUDA-core path
    const size_t state_bytes = a.bf16 ? 2 : 4;
    size_t off = 0;
    l.states_f = off;
    off = align_up(off + nstate * state_bytes);
    l.states_b = off;
    off = align_up(off + nstate * state_bytes);
    l.alpha = off;
    off = align_up(off + (size_t)a.batch * a.nh * a.nchunks * sizeof(float));
    l.h_init = off;
    if (a.review) off = align_up(off + (size_t)kHinitParts * a.batch * a.nh * a.P * a.Ns * sizeof(float));
    l.pooled = off;
    if (a.review)
        off = align_up(off + (size_t)a.batch * a.pool_splits * a.Np *
                                 ((size_t)a.nh * a.P + a.nh + (size_t)a.G * a.Ns) * sizeof(float));
    // tensor-core path: dt of every chunk in scan order (chunk_state -> chunk_out)
    l.dt_scan = off;
    if (a.bf16) off = align_up(off + (size_t)a.batch * a.nh * a.nchunks * a.Q * sizeof(float));
    l.total = off;
    return l;
}

// shape checks of the front-end; fills a (pointers left null) and the workspace split
int front_shape(int T, int H, int W, int scan_mode, const mate_frontend_dims *d, FrontArgs &a, size_t &ws_pre,
                size_t &ws_total)
{
    if (!d || T <= 0 || H <= 0 || W <= 0 || d->batch <= 0 || d->d_model <= 0 || d->nheads <= 0 || d->headdim <= 0 ||
        d->ngroups <= 0 || d->dstate <= 0)
        return MATE_ERR_INVALID_ARG;
    if (scan_mode < 0 || scan_mode > MATE_SCAN_ZZ) return MATE_ERR_INVALID_ARG;
    const int64_t N = (int64_t)T * H * W;
    if (N >= ((int64_t)1 << 31) || N * d->batch >= ((int64_t)1 << 31)) return MATE_ERR_INVALID_ARG;
    if (d->nheads % d->ngroups) return MATE_ERR_INVALID_ARG;
    if (d->dtype != MATE_BF16) return MATE_ERR_UNSUPPORTED;
    memset(&a, 0, sizeof(a));
    a.batch = d->batch;
    a.T = T;
    a.H = H;
    a.W = W;
    a.N = (int)N;
    a.mode = scan_mode;
    a.d_model = d->d_model;
    a.nh = d->nheads;
    a.d_inner = d->nheads * d->headdim;
    a.G = d->ngroups;
    a.Ns = d->dstate;
    a.dc = a.d_inner + 2 * a.G * a.Ns;
    a.dT = make_fastdiv(T);
    a.dH = make_fastdiv(H);
    a.dW = make_fastdiv(W);
    a.dHW = make_fastdiv((uint32_t)(H * W));
    if (!front_supported(a) || a.nh % 8) return MATE_ERR_UNSUPPORTED;
    // the conv addresses a token row of a batch element in 32 bits
    if (N * a.dc >= ((int64_t)1 << 31)) return MATE_ERR_UNSUPPORTED;
    const size_t M = (size_t)a.batch * a.N;
    ws_pre = align_up(M * a.dc * 2);
    ws_total = ws_pre + align_up(M * a.nh * 2);
    return MATE_OK;
}


}  // namespace mate

using namespace mate;

extern "C" {

size_t mate_bissd_workspace_bytes(int T, int H, int W, const int review_pool[3], const mate_ssd_dims *d)
{
    SsdArgs a;
    if (ssd_shape(T, H, W, review_pool, d, MATE_SCAN_SR, a) != MATE_OK) return 0;
    if (ssd_path(a) < 0) return 0;
    return ssd_workspace_layout(a).total;
}

int mate_bissd_fwd(const void *x, const float *dt, const float *A, const void *B, const void *C, const float *D,
                   int T, int H, int W, int scan_mode, const int review_pool[3], void *out, const mate_ssd_dims *d,
                   void *workspace, size_t ws_bytes, void *stream)
{
    SsdArgs a;
    int rc = ssd_shape(T, H, W, review_pool, d, scan_mode, a);
    if (rc != MATE_OK) return rc;
    const int path = ssd_path(a);
    if (path < 0) return MATE_ERR_UNSUPPORTED;
    if (!x || !dt || !A || !B || !C || !D || !out) return MATE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(out, 16) || !aligned(dt, 4) ||
        !aligned(A, 4) || !aligned(D, 4))
        return MATE_ERR_INVALID_ARG;
    const size_t e = a.bf16 ? 2 : 4;
    const size_t ntok = (size_t)a.batch * a.N;
    const size_t xbytes = ntok * a.nh * a.P * e, bbytes = ntok * a.G * a.Ns * e;
    if (overlaps(out, xbytes, x, xbytes) || overlaps(out, xbytes, B, bbytes) || overlaps(out, xbytes, C, bbytes) ||
        overlaps(out, xbytes, dt, ntok * a.nh * 4) || overlaps(out, xbytes, A, a.nh * 4) ||
        overlaps(out, xbytes, D, a.nh * 4))
        return MATE_ERR_INVALID_ARG;
    const SsdWorkspace l = ssd_workspace_layout(a);
    if (!workspace || ws_bytes < l.total || !aligned(workspace, kAlign)) return MATE_ERR_WORKSPACE;
    if (overlaps(workspace, l.total, out, xbytes) || overlaps(workspace, l.total, x, xbytes))
        return MATE_ERR_INVALID_ARG;
    a.x = x;
    a.dt = dt;
    a.A = A;
    a.B = B;
    a.C = C;
    a.D = D;
    a.out = out;
    carve(a, workspace);
    a.err = error_word_ptr();
    if (!a.err) return MATE_ERR_CUDA;
    const cudaError_t err = path == 1 ? launch_ssd_tc(a, static_cast<cudaStream_t>(stream))
                                      : launch_ssd_generic(a, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MATE_OK : MATE_ERR_CUDA;
}

int tesa_fwd(const void *q, const void *k, const void *v, int T, int H, int W, int Tw, int Sw, const int shift[3],
             void *out, const mate_attn_dims *d, void *stream)
{
    TesaArgs a;
    int rc = attn_shape(T, H, W, Tw, Sw, shift, d, a);
    if (rc != MATE_OK) return rc;
    if (a.d != 16 && a.d != 32 && a.d != 64 && a.d != 128) return MATE_ERR_UNSUPPORTED;
    const size_t e = a.bf16 ? 2 : 4;
    const size_t maxm = (size_t)Tw * Sw * Sw;
    if (maxm > 512 || 2 * maxm * a.d * e + maxm * 4 > kMaxSmem) return MATE_ERR_UNSUPPORTED;
    // bf16 storage runs on the tensor-core kernel, fp32 storage on the CUDA-core kernel
    if (a.bf16 && !tesa_tc_supported(a)) return MATE_ERR_UNSUPPORTED;
    if (!q || !k || !v || !out) return MATE_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16)) return MATE_ERR_INVALID_ARG;
    const size_t bytes = (size_t)a.batch * a.N * a.nh * a.d * e;
    if (overlaps(out, bytes, q, bytes) || overlaps(out, bytes, k, bytes) || overlaps(out, bytes, v, bytes))
        return MATE_ERR_INVALID_ARG;
    a.q = q;
    a.k = k;
    a.v = v;
    a.out = out;
    a.err = error_word_ptr();
    if (!a.err) return MATE_ERR_CUDA;
    cudaError_t err = a.bf16 ? launch_tesa_tc(a, static_cast<cudaStream_t>(stream))
                             : launch_tesa_generic(a, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MATE_OK : MATE_ERR_CUDA;
}

int mate_compose_fwd(const void *y_ma, const void *y_te, const void *w_ma, const void *w_te, void *out,
                     const mate_compose_dims *d, void *stream)
{
    if (!d) return MATE_ERR_INVALID_ARG;
    if (d->tokens <= 0 || d->k_ma < 0 || d->k_te < 0 || d->d_model <= 0 || d->k_ma + d->k_te <= 0)
        return MATE_ERR_INVALID_ARG;
    if (d->dtype != MATE_BF16) return MATE_ERR_UNSUPPORTED;
    ComposeArgs a;
    a.M = d->tokens;
    a.N = d->d_model;
    a.K1 = d->k_ma;
    a.K2 = d->k_te;
    if (a.N % 64 || !compose_tc_supported(a)) return MATE_ERR_UNSUPPORTED;
    if (!out || (a.K1 && (!y_ma || !w_ma)) || (a.K2 && (!y_te || !w_te))) return MATE_ERR_INVALID_ARG;
    const void *ptrs[5] = {y_ma, y_te, w_ma, w_te, out};
    for (const void *p : ptrs)
        if (p && !aligned(p, 16)) return MATE_ERR_INVALID_ARG;
    const size_t ob = (size_t)a.M * a.N * 2;
    if ((a.K1 && (overlaps(out, ob, y_ma, (size_t)a.M * a.K1 * 2) || overlaps(out, ob, w_ma, (size_t)a.N * a.K1 * 2))) ||
        (a.K2 && (overlaps(out, ob, y_te, (size_t)a.M * a.K2 * 2) || overlaps(out, ob, w_te, (size_t)a.N * a.K2 * 2))))
        return MATE_ERR_INVALID_ARG;
    a.y1 = y_ma;
    a.y2 = y_te;
    a.w1 = w_ma;
    a.w2 = w_te;
    a.out = out;
    a.err = error_word_ptr();
    if (!a.err) return MATE_ERR_CUDA;
    return launch_compose_tc(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MATE_OK : MATE_ERR_CUDA;
}


int mate_gate_norm_fwd(const void *y, const void *z, const float *w, float eps, void *out,
                       const mate_gate_norm_dims *d, void *stream)
{
    if (!d) return MATE_ERR_INVALID_ARG;
    if (d->tokens <= 0 || d->channels <= 0 || d->group <= 0 || !(eps >= 0.f) || !isfinite(eps))
        return MATE_ERR_INVALID_ARG;
    if (d->dtype != MATE_BF16) return MATE_ERR_UNSUPPORTED;
    GateNormArgs a;
    a.M = d->tokens;
    a.C = d->channels;
    a.group = d->group;
    a.eps = eps;
    if (!gate_norm_supported(a)) return MATE_ERR_UNSUPPORTED;
    if (!y || !z || !w || !out) return MATE_ERR_INVALID_ARG;
    const void *ptrs[4] = {y, z, w, out};
    for (const void *p : ptrs)
        if (!aligned(p, 16)) return MATE_ERR_INVALID_ARG;
    const size_t rb = (size_t)a.M * a.C * 2;
    if (overlaps(out, rb, y, rb) || overlaps(out, rb, z, rb) || overlaps(out, rb, w, (size_t)a.C * 4))
        return MATE_ERR_INVALID_ARG;
    a.y = y;
    a.z = z;
    a.w = w;
    a.out = out;
    return launch_gate_norm(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MATE_OK : MATE_ERR_CUDA;
}

size_t mate_frontend_workspace_bytes(int T, int H, int W, const mate_frontend_dims *d)
{
    FrontArgs a;
    size_t pre = 0, total = 0;
    if (front_shape(T, H, W, MATE_SCAN_SR, d, a, pre, total) != MATE_OK) return 0;
    return total;
}

int mate_frontend_fwd(const void *u, const void *w_in, const float *conv_w, const float *conv_b, const float *dt_bias,
                      int T, int H, int W, int scan_mode, void *z, void *x, float *dt, void *B, void *C,
                      const mate_frontend_dims *d, void *workspace, size_t ws_bytes, void *stream)
{
    FrontArgs a;
    size_t pre = 0, total = 0;
    int rc = front_shape(T, H, W, scan_mode, d, a, pre, total);
    if (rc != MATE_OK) return rc;
    if (!u || !w_in || !conv_w || !conv_b || !dt_bias || !z || !x || !dt || !B || !C) return MATE_ERR_INVALID_ARG;
    const void *bf[7] = {u, w_in, z, x, B, C, workspace};
    for (const void *p : bf)
        if (p && !aligned(p, 16)) return MATE_ERR_INVALID_ARG;
    if (!aligned(conv_w, 4) || !aligned(conv_b, 4) || !aligned(dt_bias, 4) || !aligned(dt, 4))
        return MATE_ERR_INVALID_ARG;
    if (!workspace || ws_bytes < total || !aligned(workspace, 256)) return MATE_ERR_WORKSPACE;
    const size_t M = (size_t)a.batch * a.N;
    const size_t ub = M * a.d_model * 2, wb = (size_t)(a.d_inner + a.dc + a.nh) * a.d_model * 2;
    const size_t zb = M * a.d_inner * 2, bb = M * a.G * a.Ns * 2, db = M * a.nh * 4;
    // every output disjoint from every input, from the workspace and from the other outputs
    const struct {
        const void *p;
        size_t n;
    } outs[5] = {{z, zb}, {x, zb}, {B, bb}, {C, bb}, {dt, db}},
      ins[6] = {{u, ub}, {w_in, wb}, {conv_w, (size_t)a.dc * 16}, {conv_b, (size_t)a.dc * 4},
                {dt_bias, (size_t)a.nh * 4}, {workspace, total}};
    for (int i = 0; i < 5; ++i) {
        for (int j = 0; j < 6; ++j)
            if (overlaps(outs[i].p, outs[i].n, ins[j].p, ins[j].n)) return MATE_ERR_INVALID_ARG;
        for (int j = i + 1; j < 5; ++j)
            if (overlaps(outs[i].p, outs[i].n, outs[j].p, outs[j].n)) return MATE_ERR_INVALID_ARG;
    }
    a.u = u;
    a.w_in = w_in;
    a.conv_w = conv_w;
    a.conv_b = conv_b;
    a.dt_bias = dt_bias;
    a.z = z;
    a.x = x;
    a.B = B;
    a.C = C;
    a.dt = dt;
    a.xbc_pre = workspace;
    a.dt_pre = static_cast<char *>(workspace) + pre;
    a.err = error_word_ptr();
    if (!a.err) return MATE_ERR_CUDA;
    return launch_front(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? MATE_OK : MATE_ERR_CUDA;
}

int mate_debug_rms_map(int T, int H, int W, int scan_mode, int flip, int32_t *out_dev, void *stream)
{
    if (T <= 0 || H <= 0 || W <= 0 || scan_mode < 0 || scan_mode > MATE_SCAN_ZZ || !out_dev)
        return MATE_ERR_INVALID_ARG;
    if ((int64_t)T * H * W >= ((int64_t)1 << 31)) return MATE_ERR_INVALID_ARG;
    cudaError_t err = launch_rms_map(T, H, W, scan_mode, flip, out_dev, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MATE_OK : MATE_ERR_CUDA;
}

int mate_debug_fastdiv(const uint32_t *n, uint32_t *q, size_t count, uint32_t d)
{
    if ((!n || !q) && count) return MATE_ERR_INVALID_ARG;
    if (d < 1 || d >= (1u << 31)) return MATE_ERR_INVALID_ARG;
    for (size_t i = 0; i < count; ++i)
        if (n[i] >= (1u << 31)) return MATE_ERR_INVALID_ARG;
    const FastDiv f = make_fastdiv(d);
    for (size_t i = 0; i < count; ++i) q[i] = fdiv(n[i], f);
    return MATE_OK;
}

int mate_debug_tesa_map(int T, int H, int W, int Tw, int Sw, const int shift[3], int32_t *out_win_dev, void *stream)
{
    mate_attn_dims d = {1, 1, 16, MATE_F32};
    TesaArgs a;
    int rc = attn_shape(T, H, W, Tw, Sw, shift, &d, a);
    if (rc != MATE_OK) return rc;
    if (!out_win_dev) return MATE_ERR_INVALID_ARG;
    cudaError_t err = launch_tesa_map(a, out_win_dev, static_cast<cudaStream_t>(stream));
    return err == cudaSuccess ? MATE_OK : MATE_ERR_CUDA;
}

int mate_last_error(void *stream)
{
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MATE_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(int)) != cudaSuccess) return MATE_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)) != cudaSuccess) return MATE_ERR_CUDA;
    }
    return word;
}

const char *mate_status_string(int code)
{
    switch (code) {
    case MATE_OK: return "ok";
    case MATE_ERR_INVALID_ARG: return "invalid argument";
    case MATE_ERR_UNSUPPORTED: return "unsupported dims or dtype";
    case MATE_ERR_CUDA: return "CUDA error";
    case MATE_ERR_TIMEOUT: return "bounded device wait timed out";
    case MATE_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    default: return "unknown status";
    }
}

int mate_version(void) { return 100; }

void mate_set_phase_hook(mate_phase_hook fn, void *user)
{
    g_hook = fn;
    g_hook_user = user;
}

uint64_t mate_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"
