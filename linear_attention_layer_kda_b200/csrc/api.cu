// api.cu -- the C ABI declared in include/kda_decode.h: handle, validation, dispatch.
#include <stdio.h>
#include <string.h>

#include <map>
#include <mutex>
#include <new>
#include <string>

#include "common.cuh"
#include "fused.cuh"
#include "prefill_gemm.cuh"
#include "status.h"

struct kda_handle_s {
    kda_config cfg{};
    int device = -1;
    int num_sms = 0;
    cudaStream_t stream = nullptr;
    void *scratch_base = nullptr;
    size_t scratch_bytes = 0;
    kda::Scratch s;
    int *status_host = nullptr;  // mapped pinned status word, readable without a sync
    int *status = nullptr;       // its device alias; kernels record KDA_ERR_DEVICE_TIMEOUT here
    void *x_stage = nullptr;    // device staging of x for kda_decode_step_host
    void *out_stage = nullptr;  // device staging of out for kda_decode_step_host
    // kda_decode_step_host_async: two staging slots, copy streams in and out and their events
    // (created on first use)
    void *hx[2] = {}, *hout[2] = {};
    cudaStream_t cstream = nullptr, ostream = nullptr;
    cudaEvent_t ev_x[2] = {}, ev_k[2] = {}, ev_o[2] = {};
    int hslot = 0;
    bool host_async_ready = false;
    kda::FusedState fused;
    void *pf_ws = nullptr;   // prefill workspace (activations of every row), grown on demand
    kda::LtGemm *lt = nullptr;  // the prefill's GEMM library handle, created on first use
    size_t pf_bytes = 0;
    bool fatal = false;  // a kernel gave up draining its copies after an abort: never step again
    std::string last_error;
};

namespace {

int fail(kda_handle h, int code, const std::string &msg)
{
    if (h) h->last_error = msg;
    return code;
}

int cuda_fail(kda_handle h, cudaError_t e, const char *what)
{
    std::string m = std::string(what) + ": " + cudaGetErrorString(e);
    (void)cudaGetLastError();
    return fail(h, KDA_ERR_CUDA, m);
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int validate_config(const kda_config *c, std::string *why)
{
    if (!c) { *why = "null config"; return KDA_ERR_INVALID_ARG; }
    for (int i = 0; i < 8; ++i)
        if (c->reserved[i] != 0) { *why = "kda_config.reserved must be zero"; return KDA_ERR_INVALID_ARG; }
    if (c->out_dtype != KDA_OUT_F32 && c->out_dtype != KDA_OUT_BF16) { *why = "bad out_dtype"; return KDA_ERR_INVALID_ARG; }
    if (c->engine < KDA_ENGINE_AUTO || c->engine > KDA_ENGINE_FUSED) { *why = "bad engine"; return KDA_ERR_INVALID_ARG; }
    if (c->max_batch < 1 || c->max_batch > 256) { *why = "max_batch must be in [1, 256]"; return KDA_ERR_INVALID_ARG; }
    if (c->hidden <= 0 || c->hidden % 128 != 0 || c->hidden > 65536) { *why = "hidden must be a positive multiple of 128 (<= 65536)"; return KDA_ERR_UNSUPPORTED_SHAPE; }
    if (c->head_dk != 64 && c->head_dk != 128) { *why = "head_dk must be 64 or 128"; return KDA_ERR_UNSUPPORTED_SHAPE; }
    if (c->head_dv != 64 && c->head_dv != 128) { *why = "head_dv must be 64 or 128"; return KDA_ERR_UNSUPPORTED_SHAPE; }
    if (c->num_heads < 1 || c->num_heads > 512) { *why = "num_heads must be in [1, 512]"; return KDA_ERR_UNSUPPORTED_SHAPE; }
    if ((c->num_heads * c->head_dk) % 128 != 0 || (c->num_heads * c->head_dv) % 128 != 0) {
        *why = "num_heads*head_dk and num_heads*head_dv must be multiples of 128";
        return KDA_ERR_UNSUPPORTED_SHAPE;
    }
    if (c->alpha_rank < 16 || c->alpha_rank > 256 || c->alpha_rank % 16 != 0) {
        *why = "alpha_rank must be a multiple of 16 in [16, 256]";
        return KDA_ERR_UNSUPPORTED_SHAPE;
    }
    return KDA_OK;
}

// Scratch layout: the simple engine's fp32 activations, then the fused engine's area.
size_t simple_scratch_bytes(const kda_config &c)
{
    const size_t B = (size_t)c.max_batch, Dk = (size_t)c.num_heads * c.head_dk, Dv = (size_t)c.num_heads * c.head_dv;
    size_t n = 0;
    n += align_up(B * Dk * 4, 256) * 3;            // q, k, z
    n += align_up(B * Dv * 4, 256) * 2;            // v, o
    n += align_up(B * (size_t)c.num_heads * 4, 256);  // bpre
    n += align_up(B * (size_t)c.alpha_rank * 4, 256); // t
    return n;
}

size_t staging_bytes(const kda_config &c)
{
    return align_up((size_t)c.max_batch * c.hidden * 2, 256) + align_up((size_t)c.max_batch * c.hidden * 4, 256);
}

kda::Dims dims_of(const kda_config &c, int B)
{
    return kda::Dims{B, c.hidden, c.num_heads, c.head_dk, c.head_dv, c.alpha_rank};
}

int pick_engine(kda_handle h, int batch)
{
    if (h->cfg.engine == KDA_ENGINE_SIMPLE) return KDA_ENGINE_SIMPLE;
    if (h->fused.bytes && kda::fused_supports(dims_of(h->cfg, batch), h->num_sms)) return KDA_ENGINE_FUSED;
    return KDA_ENGINE_SIMPLE;
}

// Engine of a multi-token step: the fused kernel while it covers batch * tokens rows and
// at most fused_max_tokens() tokens per sequence.
int tokens_engine(kda_handle h, int batch, int tokens)
{
    if (tokens == 1) return pick_engine(h, batch);
    if (tokens > kda::fused_max_tokens()) return KDA_ENGINE_SIMPLE;
    return pick_engine(h, batch * tokens);
}

int check_weights(kda_handle h, const kda_weights *w)
{
    if (!w) return fail(h, KDA_ERR_INVALID_ARG, "null weights");
    const void *p[11] = {w->wq, w->wk, w->wv, w->wo, w->sq, w->sk, w->sv, w->so, w->wa_down, w->wa_up, w->wb};
    static const char *names[11] = {"wq", "wk", "wv", "wo", "sq", "sk", "sv", "so", "wa_down", "wa_up", "wb"};
    for (int i = 0; i < 11; ++i) {
        if (!p[i]) return fail(h, KDA_ERR_INVALID_ARG, std::string("null weight pointer ") + names[i]);
        if (!aligned16(p[i])) return fail(h, KDA_ERR_INVALID_ARG, std::string("weight pointer not 16-byte aligned: ") + names[i]);
    }
    return KDA_OK;
}

bool overlaps(const void *a, size_t na, const void *b, size_t nb)
{
    const char *pa = static_cast<const char *>(a), *pb = static_cast<const char *>(b);
    return pa < pb + nb && pb < pa + na;
}

// Host-side checks shared by both step entry points (device pointers only).
int check_step(kda_handle h, const void *x, const kda_weights *w, const float *state, const void *out, int batch)
{
    if (batch < 1 || batch > h->cfg.max_batch)
        return fail(h, KDA_ERR_INVALID_ARG, "batch must be in [1, max_batch]");
    if (!x || !state || !out) return fail(h, KDA_ERR_INVALID_ARG, "null x, state or out");
    if (!aligned16(x) || !aligned16(state) || !aligned16(out))
        return fail(h, KDA_ERR_INVALID_ARG, "x, state and out must be 16-byte aligned");
    int rc = check_weights(h, w);
    if (rc) return rc;
    const kda_config &c = h->cfg;
    const size_t nx = (size_t)batch * c.hidden * 2;
    const size_t ns = (size_t)batch * c.num_heads * c.head_dk * c.head_dv * 4;
    const size_t no = (size_t)batch * c.hidden * (c.out_dtype == KDA_OUT_BF16 ? 2 : 4);
    if (overlaps(state, ns, x, nx) || overlaps(state, ns, out, no))
        return fail(h, KDA_ERR_INVALID_ARG, "state_inout overlaps x or out");
    return KDA_OK;
}

// Reads and clears the mapped status words (after the stream is idle, or to peek).  After a
// timeout the counters of the aborted step are inconsistent, so the next step resets them.
int take_device_status(kda_handle h)
{
    std::string msg;
    const int st = kda::take_status(h->status_host, &h->fatal, &msg);
    if (st == KDA_OK) return KDA_OK;
    h->fused.needs_reset = true;
    return fail(h, st, msg);
}

// Work is enqueued on the current device: it must be the handle's.
int check_device(kda_handle h)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(h, KDA_ERR_NO_DEVICE, "no current CUDA device");
    }
    if (dev != h->device) return fail(h, KDA_ERR_INVALID_ARG, "the handle's device is not the current device");
    return KDA_OK;
}

// A handle whose kernel could not drain its own copies after an abort is never used again.
int check_fatal(kda_handle h)
{
    if (!h->fatal) return KDA_OK;
    return fail(h, KDA_ERR_DEVICE_TIMEOUT, "handle unusable: an aborted step did not drain its copies in flight");
}

// Before enqueueing work: the handle is usable and its device is current.
int check_usable(kda_handle h)
{
    if (int rc = check_fatal(h)) return rc;
    return check_device(h);
}

// A tensor-parallel handle runs only fused steps, and only once every peer is mapped.
int check_tp(kda_handle h, int engine)
{
    if (!h->fused.tp_world) return KDA_OK;
    if (engine != KDA_ENGINE_FUSED)
        return fail(h, KDA_ERR_UNSUPPORTED_SHAPE, "tensor parallelism needs the fused engine for this step");
    if (!h->fused.tp_ready) return fail(h, KDA_ERR_INVALID_ARG, "tensor-parallel peers are not all mapped");
    return KDA_OK;
}

int enqueue_step(kda_handle h, const void *x, const kda_weights *w, float *state, void *out, int batch)
{
    const kda::Dims d = dims_of(h->cfg, batch);
    if (int rc = check_tp(h, pick_engine(h, batch))) return rc;
    cudaError_t e;
    if (pick_engine(h, batch) == KDA_ENGINE_FUSED)
        e = kda::fused_step(d, 1, *w, x, state, out, h->cfg.out_dtype, h->fused, h->s, h->status, h->stream);
    else
        e = kda::simple_step(d, *w, x, state, out, h->cfg.out_dtype, h->s, h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "kernel launch");
    return KDA_OK;
}

// ---------------------------------------------------------------- no-alloc entry point

// The only device memory kda_decode_step_noalloc uses besides the caller's buffers: one
// fixed array per device, for callers that may not allocate (see the header).
__device__ __align__(256) unsigned char g_noalloc_scratch[KDA_NOALLOC_MAX_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
std::map<void *, void *> g_noalloc_ptr;  // device address of the array, per CUDA context (set-up cache)

typedef CUresult (*PFN_ctxGetCurrent)(CUcontext *);

// The CUDA context current on this thread (the runtime binds the device's primary context on
// first use; cudaSetDevice does that without allocating), or null.
CUcontext current_context(int dev)
{
    static PFN_ctxGetCurrent fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_ctxGetCurrent>(p);
        else
            (void)cudaGetLastError();
    });
    if (!fn) return nullptr;
    CUcontext ctx = nullptr;
    if (fn(&ctx) != CUDA_SUCCESS) return nullptr;
    if (!ctx) {
        if (cudaSetDevice(dev) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        if (fn(&ctx) != CUDA_SUCCESS) return nullptr;
    }
    return ctx;
}

// Activations of `batch` sequences inside the array (same order as a handle's scratch);
// returns false if they do not fit.
bool noalloc_layout(const kda_config &c, int batch, char *base, kda::Scratch *s)
{
    const size_t B = (size_t)batch, Dk = (size_t)c.num_heads * c.head_dk, Dv = (size_t)c.num_heads * c.head_dv;
    const size_t sizes[7] = {B * Dk * 4, B * Dk * 4, B * Dk * 4, B * Dv * 4, B * Dv * 4,
                             B * (size_t)c.num_heads * 4, B * (size_t)c.alpha_rank * 4};
    float **dst[7] = {&s->q, &s->k, &s->z, &s->v, &s->o, &s->bpre, &s->t};
    size_t off = 0;
    for (int i = 0; i < 7; ++i) {
        if (off + sizes[i] > KDA_NOALLOC_MAX_SCRATCH_BYTES) return false;
        *dst[i] = reinterpret_cast<float *>(base + off);
        off += align_up(sizes[i], 256);
    }
    return true;
}

}  // namespace

extern "C" {

int kda_decode_step_noalloc(const kda_config *cfg, const void *x, const kda_weights *w, float *state_inout,
                            void *out, int batch, void *cuda_stream)
{
    if (!cfg) return KDA_ERR_INVALID_ARG;
    // only the shape and out dtype matter here: max_batch and engine are not used
    kda_config shape = *cfg;
    shape.max_batch = 1;
    shape.engine = KDA_ENGINE_AUTO;
    std::string why;
    int rc = validate_config(&shape, &why);
    if (rc) return rc;
    if (batch < 1) return KDA_ERR_INVALID_ARG;
    if (!x || !state_inout || !out) return KDA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(state_inout) || !aligned16(out)) return KDA_ERR_INVALID_ARG;
    rc = check_weights(nullptr, w);
    if (rc) return rc;
    const size_t nx = (size_t)batch * cfg->hidden * 2;
    const size_t ns = (size_t)batch * cfg->num_heads * cfg->head_dk * cfg->head_dv * 4;
    const size_t no = (size_t)batch * cfg->hidden * (cfg->out_dtype == KDA_OUT_BF16 ? 2 : 4);
    if (overlaps(state_inout, ns, x, nx) || overlaps(state_inout, ns, out, no)) return KDA_ERR_INVALID_ARG;
    kda::Scratch s;
    if (!noalloc_layout(*cfg, batch, nullptr, &s)) return KDA_ERR_UNSUPPORTED_SHAPE;  // over the fixed limit

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) { (void)cudaGetLastError(); return KDA_ERR_NO_DEVICE; }
    CUcontext ctx = current_context(dev);
    if (!ctx) return KDA_ERR_NO_DEVICE;
    void *base = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_noalloc_mu);
        auto it = g_noalloc_ptr.find(ctx);
        if (it == g_noalloc_ptr.end()) {  // set-up, once per context, with its device current
            int major = 0;
            if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
                (void)cudaGetLastError();
                return KDA_ERR_NO_DEVICE;
            }
            void *p = nullptr;
            const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
            if (e != cudaSuccess || !p) {
                (void)cudaGetLastError();
                return KDA_ERR_CUDA;
            }
            it = g_noalloc_ptr.emplace(ctx, p).first;
        }
        base = it->second;
    }
    noalloc_layout(*cfg, batch, static_cast<char *>(base), &s);
    const kda::Dims d = dims_of(*cfg, batch);
    const cudaError_t e = kda::simple_step(d, *w, x, state_inout, out, cfg->out_dtype, s,
                                           static_cast<cudaStream_t>(cuda_stream));
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

int kda_decode_abi_version(void) { return KDA_DECODE_ABI_VERSION; }

const char *kda_status_string(int s)
{
    switch (s) {
    case KDA_OK: return "KDA_OK";
    case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
    case KDA_ERR_UNSUPPORTED_SHAPE: return "KDA_ERR_UNSUPPORTED_SHAPE";
    case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
    case KDA_ERR_DEVICE_TIMEOUT: return "KDA_ERR_DEVICE_TIMEOUT";
    case KDA_ERR_NO_DEVICE: return "KDA_ERR_NO_DEVICE";
    case KDA_ERR_OUT_OF_MEMORY: return "KDA_ERR_OUT_OF_MEMORY";
    default: return "KDA_ERR_UNKNOWN";
    }
}

const char *kda_decode_last_error(kda_handle h) { return h ? h->last_error.c_str() : ""; }

int kda_decode_scratch_bytes(const kda_config *cfg, size_t *bytes)
{
    std::string why;
    int rc = validate_config(cfg, &why);
    if (rc) return rc;
    if (!bytes) return KDA_ERR_INVALID_ARG;
    int sms = 148, dev = 0;  // without a device, size for a 148-SM B200
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) sms = n;
    }
    (void)cudaGetLastError();
    *bytes = simple_scratch_bytes(*cfg) + staging_bytes(*cfg) + 256 +
             kda::fused_scratch_bytes(dims_of(*cfg, cfg->max_batch), sms);
    return KDA_OK;
}

int kda_decode_init(const kda_config *cfg, kda_handle *out_handle)
{
    if (!out_handle) return KDA_ERR_INVALID_ARG;
    *out_handle = nullptr;
    std::string why;
    int rc = validate_config(cfg, &why);
    if (rc) {
        fprintf(stderr, "kda_decode_init: %s\n", why.c_str());
        return rc;
    }
    int dev = -1, ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) { (void)cudaGetLastError(); return KDA_ERR_NO_DEVICE; }
    if (cudaGetDevice(&dev) != cudaSuccess) { (void)cudaGetLastError(); return KDA_ERR_NO_DEVICE; }
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) { (void)cudaGetLastError(); return KDA_ERR_NO_DEVICE; }
    if (prop.major != 10) return KDA_ERR_NO_DEVICE;  // the kernels are built for sm_100a only

    kda_handle h = new (std::nothrow) kda_handle_s;
    if (!h) return KDA_ERR_OUT_OF_MEMORY;
    h->cfg = *cfg;
    h->device = dev;
    h->num_sms = prop.multiProcessorCount;
    const size_t simple_b = simple_scratch_bytes(*cfg), stage_b = staging_bytes(*cfg);
    const size_t fused_b = cfg->engine == KDA_ENGINE_SIMPLE ? 0 : kda::fused_scratch_bytes(dims_of(*cfg, cfg->max_batch), h->num_sms);
    h->scratch_bytes = simple_b + stage_b + 256 + fused_b;
    cudaError_t e = cudaMalloc(&h->scratch_base, h->scratch_bytes);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        delete h;
        return KDA_ERR_OUT_OF_MEMORY;
    }
    char *p = static_cast<char *>(h->scratch_base);
    const size_t B = (size_t)cfg->max_batch, Dk = (size_t)cfg->num_heads * cfg->head_dk;
    const size_t Dv = (size_t)cfg->num_heads * cfg->head_dv;
    auto take = [&](size_t n) { char *r = p; p += align_up(n, 256); return r; };
    h->s.q = (float *)take(B * Dk * 4);
    h->s.k = (float *)take(B * Dk * 4);
    h->s.z = (float *)take(B * Dk * 4);
    h->s.v = (float *)take(B * Dv * 4);
    h->s.o = (float *)take(B * Dv * 4);
    h->s.bpre = (float *)take(B * cfg->num_heads * 4);
    h->s.t = (float *)take(B * cfg->alpha_rank * 4);
    h->x_stage = take(B * cfg->hidden * 2);
    h->out_stage = take(B * cfg->hidden * 4);
    (void)take(256);
    kda::fused_bind_scratch(dims_of(*cfg, cfg->max_batch), h->num_sms, p, fused_b, &h->fused);
    e = cudaMemset(h->scratch_base, 0, h->scratch_bytes);
    if (e == cudaSuccess) e = cudaHostAlloc((void **)&h->status_host, 256, cudaHostAllocMapped);
    if (e == cudaSuccess) {
        h->status_host[0] = KDA_OK;
        h->status_host[1] = 0;
        h->status_host[2] = 0;
        e = cudaHostGetDevicePointer((void **)&h->status, h->status_host, 0);
    }
    if (e == cudaSuccess) e = kda::fused_init(dims_of(*cfg, cfg->max_batch), &h->fused);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        if (h->status_host) cudaFreeHost(h->status_host);
        cudaFree(h->scratch_base);
        delete h;
        return KDA_ERR_CUDA;
    }
    *out_handle = h;
    return KDA_OK;
}

int kda_decode_set_stream(kda_handle h, void *stream)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    h->stream = static_cast<cudaStream_t>(stream);
    return KDA_OK;
}

int kda_tp_configure(kda_handle h, int rank, int world, void *ipc_handle_out)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    kda::FusedState &fs = h->fused;
    if (world < 1 || world > 8 || rank < 0 || rank >= world)
        return fail(h, KDA_ERR_INVALID_ARG, "need 1 <= world <= 8 and 0 <= rank < world");
    if (fs.tp_world) return fail(h, KDA_ERR_INVALID_ARG, "tensor parallelism is already configured");
    if (int rc = check_device(h)) return rc;
    if (!fs.bytes) return fail(h, KDA_ERR_UNSUPPORTED_SHAPE, "the in-kernel reduction needs the fused engine");
    const size_t H = (size_t)h->cfg.hidden, bmax = (size_t)h->cfg.max_batch;
    fs.tp_slot_bytes = 2 * world * bmax * H * 4;
    const size_t bytes = fs.tp_slot_bytes + 2 * (size_t)world * (H / 32) * 4;
    void *region = nullptr;
    cudaError_t e = cudaMalloc(&region, bytes);
    if (e == cudaSuccess) e = cudaMemset(region, 0, bytes);
    cudaIpcMemHandle_t ipc;
    if (e == cudaSuccess && world > 1) e = cudaIpcGetMemHandle(&ipc, region);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        if (region) cudaFree(region);
        return cuda_fail(h, e, "exchange region");
    }
    if (ipc_handle_out && world > 1) memcpy(ipc_handle_out, &ipc, sizeof ipc);
    fs.tp_world = world;
    fs.tp_rank = rank;
    fs.tp_bmax = (int)bmax;
    fs.tp_region[rank] = region;
    fs.tp_ready = world == 1;
    return KDA_OK;
}

int kda_tp_set_peer(kda_handle h, int peer, const void *ipc_handle)
{
    if (!h || !ipc_handle) return KDA_ERR_INVALID_ARG;
    kda::FusedState &fs = h->fused;
    if (!fs.tp_world) return fail(h, KDA_ERR_INVALID_ARG, "tensor parallelism is not configured");
    if (peer < 0 || peer >= fs.tp_world || peer == fs.tp_rank) return fail(h, KDA_ERR_INVALID_ARG, "bad peer rank");
    if (fs.tp_region[peer]) return fail(h, KDA_ERR_INVALID_ARG, "peer already mapped");
    if (int rc = check_device(h)) return rc;
    cudaIpcMemHandle_t ipc;
    memcpy(&ipc, ipc_handle, sizeof ipc);
    void *p = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&p, ipc, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) return cuda_fail(h, e, "mapping a peer's exchange region");
    fs.tp_region[peer] = p;
    bool all = true;
    for (int r = 0; r < fs.tp_world; ++r) all = all && fs.tp_region[r];
    fs.tp_ready = all;
    return KDA_OK;
}

int kda_decode_set_launch_overlap(kda_handle h, int on)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    h->fused.overlap = on != 0;
    return KDA_OK;
}

int kda_decode_engine(kda_handle h, int batch)
{
    if (!h || batch < 1 || batch > h->cfg.max_batch) return -KDA_ERR_INVALID_ARG;
    return pick_engine(h, batch);
}

int kda_decode_tokens_engine(kda_handle h, int batch, int tokens)
{
    if (!h || batch < 1 || tokens < 1 || (long long)batch * tokens > h->cfg.max_batch) return -KDA_ERR_INVALID_ARG;
    return tokens_engine(h, batch, tokens);
}

int kda_decode_launches_per_step(kda_handle h, int batch)
{
    if (!h || batch < 1 || batch > h->cfg.max_batch) return -KDA_ERR_INVALID_ARG;
    if (pick_engine(h, batch) == KDA_ENGINE_FUSED) return kda::fused_launches();
    return h->cfg.head_dk == h->cfg.head_dv ? kda::simple_launches() : kda::simple_launches() + 1;
}

int kda_decode_step(kda_handle h, const void *x, const kda_weights *w, float *state_inout, void *out, int batch)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    int rc = check_usable(h);
    if (rc) return rc;
    rc = check_step(h, x, w, state_inout, out, batch);
    if (rc) return rc;
    // A timeout recorded by an earlier step is reported (and cleared) here.
    rc = take_device_status(h);
    if (rc) return rc;
    return enqueue_step(h, x, w, state_inout, out, batch);
}

int kda_decode_step_host(kda_handle h, const void *x_host, const kda_weights *w, float *state_inout,
                         void *out_host, int batch)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    if (!x_host || !out_host) return fail(h, KDA_ERR_INVALID_ARG, "null host buffer");
    int rc = check_usable(h);
    if (rc) return rc;
    rc = check_step(h, h->x_stage, w, state_inout, h->out_stage, batch);
    if (rc) return rc;
    rc = take_device_status(h);
    if (rc) return rc;
    const size_t nx = (size_t)batch * h->cfg.hidden * 2;
    const size_t no = (size_t)batch * h->cfg.hidden * (h->cfg.out_dtype == KDA_OUT_BF16 ? 2 : 4);
    cudaError_t e = cudaMemcpyAsync(h->x_stage, x_host, nx, cudaMemcpyHostToDevice, h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "copying x to the device");
    rc = enqueue_step(h, h->x_stage, w, state_inout, h->out_stage, batch);
    if (rc) return rc;
    e = cudaMemcpyAsync(out_host, h->out_stage, no, cudaMemcpyDeviceToHost, h->stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "copying out to the host");
    return take_device_status(h);
}

static int host_async_setup(kda_handle h)
{
    if (h->host_async_ready) return KDA_OK;
    // each resource is created once: a call after a failed set-up creates only what is missing
    const size_t B = (size_t)h->cfg.max_batch, H = (size_t)h->cfg.hidden;
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        if (!h->hx[i]) e = cudaMalloc(&h->hx[i], B * H * 2);
        if (e == cudaSuccess && !h->hout[i]) e = cudaMalloc(&h->hout[i], B * H * 4);
        if (e == cudaSuccess && !h->ev_x[i]) e = cudaEventCreateWithFlags(&h->ev_x[i], cudaEventDisableTiming);
        if (e == cudaSuccess && !h->ev_k[i]) e = cudaEventCreateWithFlags(&h->ev_k[i], cudaEventDisableTiming);
        if (e == cudaSuccess && !h->ev_o[i]) e = cudaEventCreateWithFlags(&h->ev_o[i], cudaEventDisableTiming);
    }
    if (e == cudaSuccess && !h->cstream) e = cudaStreamCreateWithFlags(&h->cstream, cudaStreamNonBlocking);
    if (e == cudaSuccess && !h->ostream) e = cudaStreamCreateWithFlags(&h->ostream, cudaStreamNonBlocking);
    // the slots start free: their "step done" and "out copied" events complete at once
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaEventRecord(h->ev_k[i], h->cstream);
        if (e == cudaSuccess) e = cudaEventRecord(h->ev_o[i], h->ostream);
    }
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return fail(h, KDA_ERR_OUT_OF_MEMORY, "host-step staging allocation failed");
    }
    h->host_async_ready = true;
    return KDA_OK;
}

int kda_decode_step_host_async(kda_handle h, const void *x_host, const kda_weights *w, float *state_inout,
                               void *out_host, int batch)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    if (!x_host || !out_host) return fail(h, KDA_ERR_INVALID_ARG, "null host buffer");
    int rc = check_usable(h);
    if (rc) return rc;
    rc = host_async_setup(h);
    if (rc) return rc;
    const int s = h->hslot;
    rc = check_step(h, h->hx[s], w, state_inout, h->hout[s], batch);
    if (rc) return rc;
    rc = take_device_status(h);
    if (rc) return rc;
    const size_t nx = (size_t)batch * h->cfg.hidden * 2;
    const size_t no = (size_t)batch * h->cfg.hidden * (h->cfg.out_dtype == KDA_OUT_BF16 ? 2 : 4);
    // in: once the step that last used slot s has read its x; the step: once x is in and the
    // slot's previous out has been copied back; out: once the step is done
    cudaError_t e = cudaStreamWaitEvent(h->cstream, h->ev_k[s], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(h->hx[s], x_host, nx, cudaMemcpyHostToDevice, h->cstream);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_x[s], h->cstream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->stream, h->ev_x[s], 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->stream, h->ev_o[s], 0);
    if (e != cudaSuccess) return cuda_fail(h, e, "copying x to the device");
    rc = enqueue_step(h, h->hx[s], w, state_inout, h->hout[s], batch);
    if (rc) return rc;
    e = cudaEventRecord(h->ev_k[s], h->stream);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->ostream, h->ev_k[s], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(out_host, h->hout[s], no, cudaMemcpyDeviceToHost, h->ostream);
    if (e == cudaSuccess) e = cudaEventRecord(h->ev_o[s], h->ostream);
    if (e != cudaSuccess) return cuda_fail(h, e, "copying out to the host");
    h->hslot = s ^ 1;
    return KDA_OK;
}

int kda_decode_step_tokens(kda_handle h, const void *x, const kda_weights *w, float *state_inout, void *out,
                           int batch, int tokens)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    if (tokens < 1) return fail(h, KDA_ERR_INVALID_ARG, "tokens must be >= 1");
    if (int rc0 = check_usable(h)) return rc0;
    if (tokens == 1) return kda_decode_step(h, x, w, state_inout, out, batch);
    if (batch < 1 || (long long)batch * tokens > h->cfg.max_batch)
        return fail(h, KDA_ERR_INVALID_ARG, "batch * tokens must be in [1, max_batch]");
    if (!x || !state_inout || !out) return fail(h, KDA_ERR_INVALID_ARG, "null x, state or out");
    if (!aligned16(x) || !aligned16(state_inout) || !aligned16(out))
        return fail(h, KDA_ERR_INVALID_ARG, "x, state and out must be 16-byte aligned");
    int rc = check_weights(h, w);
    if (rc) return rc;
    const kda_config &c = h->cfg;
    const size_t rows = (size_t)batch * tokens;
    const size_t nx = rows * c.hidden * 2, no = rows * c.hidden * (c.out_dtype == KDA_OUT_BF16 ? 2 : 4);
    const size_t ns = (size_t)batch * c.num_heads * c.head_dk * c.head_dv * 4;
    if (overlaps(state_inout, ns, x, nx) || overlaps(state_inout, ns, out, no))
        return fail(h, KDA_ERR_INVALID_ARG, "state_inout overlaps x or out");
    rc = take_device_status(h);
    if (rc) return rc;
    if (int rc1 = check_tp(h, tokens_engine(h, batch, tokens))) return rc1;
    cudaError_t e;
    if (tokens_engine(h, batch, tokens) == KDA_ENGINE_FUSED)
        e = kda::fused_step(dims_of(c, batch * tokens), tokens, *w, x, state_inout, out, c.out_dtype, h->fused, h->s,
                            h->status, h->stream);
    else
        e = kda::simple_step_tokens(dims_of(c, batch), tokens, *w, x, state_inout, out, c.out_dtype, h->s, h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "kernel launch");
    return KDA_OK;
}

int kda_prefill(kda_handle h, const void *x, const kda_weights *w, float *state_inout, void *out, int batch,
                int tokens, int chunk)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    if (int rc0 = check_usable(h)) return rc0;
    const kda_config &c = h->cfg;
    if (chunk == 0) chunk = 32;
    if (batch < 1 || tokens < 1) return fail(h, KDA_ERR_INVALID_ARG, "batch and tokens must be >= 1");
    if (!kda::chunk_supported(c.head_dk, c.head_dv, chunk))
        return fail(h, KDA_ERR_INVALID_ARG, "chunk must be 16, 32 or 64");
    if (!x || !state_inout || !out) return fail(h, KDA_ERR_INVALID_ARG, "null x, state or out");
    if (!aligned16(x) || !aligned16(state_inout) || !aligned16(out))
        return fail(h, KDA_ERR_INVALID_ARG, "x, state and out must be 16-byte aligned");
    int rc = check_weights(h, w);
    if (rc) return rc;
    const long long rows_ll = (long long)batch * tokens;
    const size_t Dk = (size_t)c.num_heads * c.head_dk, Dv = (size_t)c.num_heads * c.head_dv;
    if (rows_ll > (1LL << 31) / (long long)(Dk > (size_t)c.hidden ? Dk : (size_t)c.hidden))
        return fail(h, KDA_ERR_INVALID_ARG, "batch * tokens too large");
    const size_t rows = (size_t)rows_ll;
    const size_t nx = rows * c.hidden * 2, no = rows * c.hidden * (c.out_dtype == KDA_OUT_BF16 ? 2 : 4);
    const size_t ns = (size_t)batch * c.num_heads * c.head_dk * c.head_dv * 4;
    if (overlaps(state_inout, ns, x, nx) || overlaps(state_inout, ns, out, no))
        return fail(h, KDA_ERR_INVALID_ARG, "state_inout overlaps x or out");
    rc = take_device_status(h);
    if (rc) return rc;
    if (!h->lt) {
        const cudaError_t e0 = kda::lt_create(&h->lt);
        if (e0 != cudaSuccess) return cuda_fail(h, e0, "GEMM library handle");
    }
    // workspace: the fp32 activations of every row, then the GEMMs' bf16 splits
    const kda::Dims d = dims_of(c, (int)rows);
    const size_t sizes[9] = {rows * Dk * 4, rows * Dk * 4, rows * Dk * 4, rows * Dv * 4, rows * Dv * 4,
                             rows * (size_t)c.num_heads * 4, rows * (size_t)c.alpha_rank * 4,
                             kda::prefill_gemm_ws_bytes(d),
                             kda::chunk_ws_bytes(c.head_dk, c.num_heads, batch, tokens, chunk)};
    size_t need = 0;
    for (size_t sz : sizes) need += align_up(sz, 256);
    if (need > h->pf_bytes) {
        if (h->pf_ws && cudaFree(h->pf_ws) != cudaSuccess) (void)cudaGetLastError();  // waits for its users
        h->pf_ws = nullptr;
        h->pf_bytes = 0;
        if (cudaMalloc(&h->pf_ws, need) != cudaSuccess) {
            (void)cudaGetLastError();
            return fail(h, KDA_ERR_OUT_OF_MEMORY, "prefill workspace allocation failed");
        }
        h->pf_bytes = need;
    }
    kda::Scratch s;
    float **dst[7] = {&s.q, &s.k, &s.z, &s.v, &s.o, &s.bpre, &s.t};
    char *p = static_cast<char *>(h->pf_ws);
    for (int i = 0; i < 7; ++i) {
        *dst[i] = reinterpret_cast<float *>(p);
        p += align_up(sizes[i], 256);
    }
    void *gws = p, *cws = p + align_up(sizes[7], 256);
    cudaError_t e = kda::prefill_projections(h->lt, d, *w, x, s, gws, h->stream);
    if (e == cudaSuccess)
        e = kda::chunk_state(d, batch, tokens, chunk, s, state_inout, cws, h->status, h->fused.timeout_ns, h->stream);
    if (e == cudaSuccess) e = kda::prefill_out_projection(h->lt, d, *w, s.o, out, c.out_dtype, gws, h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "prefill launch");
    return KDA_OK;
}

static int state_copy(kda_handle h, void *dst, const void *src, int seq0, int nseq, bool to_host)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    if (!dst || !src) return fail(h, KDA_ERR_INVALID_ARG, "null state or host buffer");
    if (seq0 < 0 || nseq < 1 || (long long)seq0 + nseq > h->cfg.max_batch)
        return fail(h, KDA_ERR_INVALID_ARG, "need seq0 >= 0, nseq >= 1 and seq0 + nseq <= max_batch");
    if (int rc = check_device(h)) return rc;
    const kda_config &c = h->cfg;
    const size_t per_seq = (size_t)c.num_heads * c.head_dk * c.head_dv * 4;
    const size_t off = (size_t)seq0 * per_seq, n = (size_t)nseq * per_seq;
    const cudaError_t e =
        to_host ? cudaMemcpyAsync(dst, static_cast<const char *>(src) + off, n, cudaMemcpyDeviceToHost, h->stream)
                : cudaMemcpyAsync(static_cast<char *>(dst) + off, src, n, cudaMemcpyHostToDevice, h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, to_host ? "state checkpoint copy" : "state restore copy");
    return KDA_OK;
}

int kda_state_checkpoint(kda_handle h, const float *state, int seq0, int nseq, void *host_dst)
{
    return state_copy(h, host_dst, state, seq0, nseq, true);
}

int kda_state_restore(kda_handle h, const void *host_src, float *state, int seq0, int nseq)
{
    return state_copy(h, state, host_src, seq0, nseq, false);
}

int kda_decode_sync(kda_handle h)
{
    if (!h) return KDA_ERR_INVALID_ARG;
    cudaError_t e = cudaStreamSynchronize(h->stream);
    if (e == cudaSuccess && h->cstream) e = cudaStreamSynchronize(h->cstream);
    if (e == cudaSuccess && h->ostream) e = cudaStreamSynchronize(h->ostream);
    if (e != cudaSuccess) return cuda_fail(h, e, "stream synchronize");
    const int st = take_device_status(h);
    return st ? st : check_fatal(h);
}

int kda_decode_debug_copy(kda_handle h, int which, void *dst, size_t bytes)
{
    if (!h || !dst) return KDA_ERR_INVALID_ARG;
    const kda_config &c = h->cfg;
    const size_t B = (size_t)c.max_batch;
    const float *src = nullptr;
    size_t n = 0;
    switch (which) {
    case KDA_DEBUG_Q: src = h->s.q; n = B * c.num_heads * c.head_dk; break;
    case KDA_DEBUG_K: src = h->s.k; n = B * c.num_heads * c.head_dk; break;
    case KDA_DEBUG_V: src = h->s.v; n = B * c.num_heads * c.head_dv; break;
    case KDA_DEBUG_BETA_PRE: src = h->s.bpre; n = B * c.num_heads; break;
    case KDA_DEBUG_T: src = h->s.t; n = B * c.alpha_rank; break;
    case KDA_DEBUG_TRACE:
        if (!h->fused.trace) return fail(h, KDA_ERR_INVALID_ARG, "library built without KDA_TRACE");
        src = reinterpret_cast<const float *>(h->fused.trace);
        n = (size_t)h->fused.num_ctas * kda::kTraceSlots * 2;
        break;
    default: return fail(h, KDA_ERR_INVALID_ARG, "unknown debug tensor");
    }
    if (bytes > n * 4) return fail(h, KDA_ERR_INVALID_ARG, "debug copy larger than the tensor");
    cudaError_t e = cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, h->stream);
    if (e != cudaSuccess) return cuda_fail(h, e, "debug copy");
    return KDA_OK;
}

int kda_decode_destroy(kda_handle h)
{
    if (!h) return KDA_OK;
    int rc = KDA_OK;
    if (cudaStreamSynchronize(h->stream) != cudaSuccess) { (void)cudaGetLastError(); rc = KDA_ERR_CUDA; }
    for (cudaStream_t cs : {h->cstream, h->ostream}) {
        if (!cs) continue;
        if (cudaStreamSynchronize(cs) != cudaSuccess) { (void)cudaGetLastError(); rc = KDA_ERR_CUDA; }
        (void)cudaStreamDestroy(cs);
    }
    for (int i = 0; i < 2; ++i) {
        if (h->ev_x[i]) (void)cudaEventDestroy(h->ev_x[i]);
        if (h->ev_k[i]) (void)cudaEventDestroy(h->ev_k[i]);
        if (h->ev_o[i]) (void)cudaEventDestroy(h->ev_o[i]);
        if (h->hx[i]) (void)cudaFree(h->hx[i]);
        if (h->hout[i]) (void)cudaFree(h->hout[i]);
    }
    kda::fused_destroy(&h->fused);
    if (h->pf_ws && cudaFree(h->pf_ws) != cudaSuccess) { (void)cudaGetLastError(); rc = KDA_ERR_CUDA; }
    kda::lt_destroy(h->lt);
    for (int r = 0; r < h->fused.tp_world; ++r) {
        void *p = h->fused.tp_region[r];
        if (!p) continue;
        const cudaError_t e = r == h->fused.tp_rank ? cudaFree(p) : cudaIpcCloseMemHandle(p);
        if (e != cudaSuccess) { (void)cudaGetLastError(); rc = KDA_ERR_CUDA; }
    }
    if (h->status_host && cudaFreeHost(h->status_host) != cudaSuccess) { (void)cudaGetLastError(); rc = KDA_ERR_CUDA; }
    if (cudaFree(h->scratch_base) != cudaSuccess) { (void)cudaGetLastError(); rc = KDA_ERR_CUDA; }
    delete h;
    return rc;
}

}  // extern "C"
