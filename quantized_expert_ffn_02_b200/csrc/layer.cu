// layer.cu -- the C ABI of libmoe.so: argument checks, workspace, launch sequencing, status.
//
// moe_forward enqueues (all on the caller's stream, no host synchronisation):
//   router logits + top-k (K2) -> bucketing (K3) -> gate/up + SiLU (K4) -> down (K4)
//   -> combine with the shared expert (K6)
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "internal.cuh"

namespace qe {

// Event pairs around launches, summed on demand.  Events are created lazily and reused.
struct Profiler {
    bool on = false;
    struct Pair { cudaEvent_t a, b; int kernel; };
    std::vector<Pair> pending;
    std::vector<cudaEvent_t> pool;
    cudaEvent_t open_ev = nullptr;
    double total_ms[MOE_KERNEL_COUNT] = {};
    int64_t count[MOE_KERNEL_COUNT] = {};

    cudaEvent_t get() {
        if (!pool.empty()) {
            cudaEvent_t e = pool.back();
            pool.pop_back();
            return e;
        }
        cudaEvent_t e = nullptr;
        cudaEventCreate(&e);
        return e;
    }
    void collect() {
        for (Pair& p : pending) {
            float ms = 0.f;
            if (cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
                total_ms[p.kernel] += ms;
                count[p.kernel] += 1;
            }
            pool.push_back(p.a);
            pool.push_back(p.b);
        }
        pending.clear();
    }
    ~Profiler() {
        for (Pair& p : pending) { cudaEventDestroy(p.a); cudaEventDestroy(p.b); }
        for (cudaEvent_t e : pool) cudaEventDestroy(e);
        if (open_ev) cudaEventDestroy(open_ev);
    }
};

void prof_mark(Profiler* p, int kernel, bool begin, cudaStream_t s) {
    if (!p || !p->on) return;
    cudaEvent_t e = p->get();
    if (!e) return;
    cudaEventRecord(e, s);
    if (begin) {
        p->open_ev = e;
    } else if (p->open_ev) {
        p->pending.push_back(Profiler::Pair{p->open_ev, e, kernel});
        p->open_ev = nullptr;
    }
}

}  // namespace qe

struct moe_layer {
    moe_config cfg;
    moe_weights w;
    qe::LayerDims dims;
    qe::Workspace ws;
    int device;
    int num_sms;
    void* ws_base;
    size_t ws_bytes;
    uint16_t* x_stage[2];  // [maxT][d] x staging for the host-buffer calls, used in turn
    void* out_stage;       // [maxT][d] output staging (when the output cannot be written in place)
    int x_next = 0;        // the x stage of the next host-buffer call
    cudaStream_t copy_s = nullptr;           // host -> device copies of x, ahead of the kernels
    cudaEvent_t x_landed[2] = {nullptr, nullptr};   // a stage's x is on the device
    cudaEvent_t x_read[2] = {nullptr, nullptr};     // the kernels that read a stage are done
    cudaStream_t last_stream;
    int last_launches;
    qe::Profiler prof;
    qe::PrefillPlan* plan = nullptr;     // TMA maps of the grouped-GEMM path (null if unsupported)
    int64_t prefill_min_tokens = 128;    // batches at least this large take the grouped-GEMM path
    int t1_mode = 0;                     // T = 1: 2 single launch, 1 single-token kernels, 0 general
    bool fused_ok = false;               // the single-launch path is usable for this layer
    bool fused2_ok = false;              // ... and for two-token batches
    bool union_mma = true;               // small batches: the tensor-core union kernels when they fit
    bool ragged = false;                 // some routed expert lives outside the contiguous [E] arrays
};

namespace {

bool aligned16(const void* p) { return ((uintptr_t)p & 15) == 0; }

// Outputs up to this size are written straight into mapped pinned host memory by the kernels.
constexpr size_t kDirectOutputBytes = 1 << 20;

moe_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    if (e == cudaErrorMemoryAllocation) return MOE_ERR_OOM;
    return MOE_ERR_CUDA;
}

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Bytes of one weight row of `cols` columns in the container (scales are separate arrays).
size_t row_bytes(int wkind, size_t cols) {
    switch (wkind) {
        case MOE_W_INT4_ROWSCALE: return cols / 2;
        case MOE_W_INT8_ROWSCALE: return cols;
        case MOE_W_INT2_ROWSCALE: return cols / 4;
        default: return cols * 2;
    }
}

__global__ void set_expert_kernel(const void** etab, int E, int e, const void* gu, const void* gus, const void* dn,
                                  const void* dns) {
    etab[e] = gu;
    etab[E + e] = gus;
    etab[2 * E + e] = dn;
    etab[3 * E + e] = dns;
}

// Carves the workspace out of one allocation.  With base == nullptr it only measures.
// max_groups > 0 adds the grouped-GEMM path's buffers.
size_t carve(const moe_config& c, size_t max_groups, char* base, qe::Workspace* ws, uint16_t** x_stage,
             void** out_stage) {   // x_stage: two buffers
    const size_t T = (size_t)c.max_tokens, E = (size_t)c.n_experts, k = (size_t)c.top_k;
    const size_t S = c.n_shared > 0 ? 1 : 0;
    const size_t fmax = S && c.f_shared > c.f ? (size_t)c.f_shared : (size_t)c.f;
    const size_t slots = T * k + T * S;
    size_t o = 0;
    auto take = [&](size_t bytes) -> char* {
        char* p = base ? base + o : nullptr;
        o = round_up(o + bytes, 256);
        return p;
    };
    qe::Workspace w{};
    w.logits = (double*)take(sizeof(double) * T * E);
    w.keys = (double*)take(sizeof(double) * std::min(T, (size_t)qe::kRouteSmallMaxT) * E);
    w.rsmall = (double*)take(sizeof(double) * qe::route_small_part_doubles((int)E, (int)T));
    w.rsmall_cnt = (unsigned int*)take(sizeof(unsigned int) * qe::route_small_groups((int)E));
    w.rsplit_n = qe::router_split_doubles((int)E, (int)T);
    w.rsplit = w.rsplit_n ? (double*)take(sizeof(double) * w.rsplit_n) : nullptr;
    w.idx = (int32_t*)take(sizeof(int32_t) * T * k);
    w.wts = (float*)take(sizeof(float) * T * k);
    w.asc = (int32_t*)take(sizeof(int32_t) * T * k);
    w.xsum = (double*)take(sizeof(double) * T);
    w.cnt = (int32_t*)take(sizeof(int32_t) * E);
    w.off = (int32_t*)take(sizeof(int32_t) * (E + 1));
    w.perm = (int32_t*)take(sizeof(int32_t) * T * k);
    w.slot_of = (int32_t*)take(sizeof(int32_t) * T * k);
    w.ulist = (int32_t*)take(sizeof(int32_t) * E);
    w.n_unique = (int32_t*)take(sizeof(int32_t));
    w.h = (uint16_t*)take(sizeof(uint16_t) * slots * fmax);
    w.Y = (float*)take(sizeof(float) * slots * (size_t)c.d);
    w.status = (int32_t*)take(sizeof(int32_t));
    w.counter = (uint32_t*)take(sizeof(uint32_t));
    w.etab = (const void**)take(sizeof(void*) * 4 * E);
    w.rpart = (double*)take(sizeof(double) * 2 * E * (c.d / 1024 > 0 ? (size_t)c.d / 1024 : 1));
    w.gbar = (unsigned long long*)take(sizeof(unsigned long long));
    w.trace = (unsigned long long*)take(sizeof(unsigned long long) * qe::kTraceCtas * qe::kTraceStamps);
    if (max_groups) {
        w.xg = (uint16_t*)take(sizeof(uint16_t) * slots * (size_t)c.d);
        w.groups = (int32_t*)take(sizeof(int32_t) * 4 * max_groups);
        w.n_groups = (int32_t*)take(sizeof(int32_t) * 2);
        w.xsum_slot = (float*)take(sizeof(float) * slots);
    }
    uint16_t* xs0 = (uint16_t*)take(sizeof(uint16_t) * T * (size_t)c.d);
    uint16_t* xs1 = (uint16_t*)take(sizeof(uint16_t) * T * (size_t)c.d);
    void* os = (void*)take(sizeof(float) * T * (size_t)c.d);
    if (ws) *ws = w;
    if (x_stage) {
        x_stage[0] = xs0;
        x_stage[1] = xs1;
    }
    if (out_stage) *out_stage = os;
    return o;
}

void destroy_streams(moe_layer* L) {
    for (int i = 0; i < 2; ++i) {
        if (L->x_landed[i]) cudaEventDestroy(L->x_landed[i]);
        if (L->x_read[i]) cudaEventDestroy(L->x_read[i]);
        L->x_landed[i] = L->x_read[i] = nullptr;
    }
    if (L->copy_s) cudaStreamDestroy(L->copy_s);
    L->copy_s = nullptr;
}

moe_status check_config(const moe_config* c, const moe_weights* w) {
    if (!c || !w) return MOE_ERR_INVALID_ARG;
    if (c->d <= 0 || c->d % 64 || c->f <= 0 || c->f % 64) return MOE_ERR_INVALID_ARG;
    if (c->n_experts < 1 || c->n_experts > 1024) return MOE_ERR_INVALID_ARG;
    if (c->top_k < 1 || c->top_k > c->n_experts || c->top_k > 32) return MOE_ERR_INVALID_ARG;
    if (c->n_shared < 0 || c->n_shared > 1) return MOE_ERR_INVALID_ARG;
    if (c->n_shared && (c->f_shared <= 0 || c->f_shared % 64)) return MOE_ERR_INVALID_ARG;
    if (c->max_tokens < 1) return MOE_ERR_INVALID_ARG;
    if (c->router != MOE_ROUTER_SOFTMAX_TOPK && c->router != MOE_ROUTER_SIGMOID_BIAS) return MOE_ERR_INVALID_ARG;
    if (c->wkind < MOE_W_INT4_ROWSCALE || c->wkind > MOE_W_INT2_ROWSCALE) return MOE_ERR_INVALID_ARG;
    if (!(c->routed_scaling_factor == c->routed_scaling_factor)) return MOE_ERR_INVALID_ARG;
    if (c->d > 14336) return MOE_ERR_UNSUPPORTED;     // router x tile must fit in shared memory
    if ((size_t)c->max_tokens * (size_t)(c->top_k + 1) > (size_t)INT32_MAX / 2) return MOE_ERR_UNSUPPORTED;
    const bool q = c->wkind != MOE_W_BF16;     // a container with per-row scales
    if (!w->router_w || !w->gate_up || !w->down) return MOE_ERR_INVALID_ARG;
    if (q && (!w->gate_up_scale || !w->down_scale)) return MOE_ERR_INVALID_ARG;
    if (c->n_shared && (!w->shared_gate_up || !w->shared_down)) return MOE_ERR_INVALID_ARG;
    if (c->n_shared && q && (!w->shared_gate_up_scale || !w->shared_down_scale)) return MOE_ERR_INVALID_ARG;
    const void* ptrs[] = {w->router_w, w->router_bias, w->gate_up, w->gate_up_scale, w->down, w->down_scale,
                          w->shared_gate_up, w->shared_gate_up_scale, w->shared_down, w->shared_down_scale};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_str(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_OOM: return "out of device memory";
        case MOE_ERR_TIMEOUT: return "device-side wait timed out";
        case MOE_ERR_RANGE: return "value out of range";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    }
    return "unknown status";
}

moe_status moe_pack_int4(const float* w, int64_t rows, int64_t cols, uint8_t* packed, float* scales,
                         moe_stream stream) {
    if (rows < 0 || cols <= 0 || (cols & 1)) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!w || !packed || !scales) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)w & 3) || ((uintptr_t)scales & 3)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int* status = nullptr;
    cudaError_t e = cudaMallocAsync((void**)&status, sizeof(int), s);
    if (e != cudaSuccess) return from_cuda(e);
    e = cudaMemsetAsync(status, 0, sizeof(int), s);
    if (e == cudaSuccess) e = qe::launch_pack_int4(w, rows, cols, packed, scales, status, s);
    int host_status = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host_status, status, sizeof(int), cudaMemcpyDeviceToHost, s);
    cudaError_t e2 = cudaFreeAsync(status, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = e2;
    if (e != cudaSuccess) return from_cuda(e);
    return host_status ? (moe_status)host_status : MOE_OK;
}

// The int8 and packed int2 tiers: the same synchronous shape as moe_pack_int4.
static moe_status pack_tier(int bits, const float* w, int64_t rows, int64_t cols, uint8_t* packed, float* scales,
                            moe_stream stream) {
    const int per_byte = 8 / bits;
    if (rows < 0 || cols <= 0 || (cols % per_byte)) return MOE_ERR_INVALID_ARG;
    if (rows == 0) return MOE_OK;
    if (!w || !packed || !scales) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)w & 3) || ((uintptr_t)scales & 3)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int* status = nullptr;
    cudaError_t e = cudaMallocAsync((void**)&status, sizeof(int), s);
    if (e != cudaSuccess) return from_cuda(e);
    e = cudaMemsetAsync(status, 0, sizeof(int), s);
    if (e == cudaSuccess) e = qe::launch_pack_tier(bits, w, rows, cols, packed, scales, status, s);
    int host_status = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&host_status, status, sizeof(int), cudaMemcpyDeviceToHost, s);
    cudaError_t e2 = cudaFreeAsync(status, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = e2;
    if (e != cudaSuccess) return from_cuda(e);
    return host_status ? (moe_status)host_status : MOE_OK;
}

moe_status moe_pack_int8(const float* w, int64_t rows, int64_t cols, int8_t* q, float* scales, moe_stream stream) {
    return pack_tier(8, w, rows, cols, reinterpret_cast<uint8_t*>(q), scales, stream);
}

moe_status moe_pack_int2(const float* w, int64_t rows, int64_t cols, uint8_t* packed, float* scales,
                         moe_stream stream) {
    return pack_tier(2, w, rows, cols, packed, scales, stream);
}

moe_status moe_layer_create(const moe_config* cfg, const moe_weights* w, moe_layer** out) {
    if (!out) return MOE_ERR_INVALID_ARG;
    moe_status st = check_config(cfg, w);
    if (st != MOE_OK) return st;
    moe_layer* L = new (std::nothrow) moe_layer();
    if (!L) return MOE_ERR_OOM;
    L->cfg = *cfg;
    L->w = *w;
    if (cfg->router != MOE_ROUTER_SIGMOID_BIAS) L->w.router_bias = nullptr;
    L->dims = qe::LayerDims{cfg->d, cfg->f, cfg->n_experts, cfg->top_k, cfg->n_shared > 0 ? 1 : 0,
                            cfg->n_shared > 0 ? cfg->f_shared : 0, cfg->router, cfg->wkind, cfg->out_bf16 ? 1 : 0,
                            cfg->routed_scaling_factor};
    cudaError_t e = cudaGetDevice(&L->device);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&L->num_sms, cudaDevAttrMultiProcessorCount, L->device);
    if (e == cudaSuccess) e = qe::prepare_router(L->dims);
    if (e == cudaSuccess) e = qe::prepare_bucket(L->dims);
    if (e == cudaSuccess) e = qe::prepare_decode(L->dims);
    if (e == cudaSuccess) e = qe::prepare_decode_mma();
    if (e == cudaSuccess) e = qe::prepare_decode_fused(L->dims, L->num_sms, &L->fused_ok, 1);
    if (e == cudaSuccess && cfg->max_tokens >= 2)
        e = qe::prepare_decode_fused(L->dims, L->num_sms, &L->fused2_ok, 2);
    const bool gemm = qe::prefill_supported(L->dims);
    if (e == cudaSuccess && gemm) e = qe::prepare_prefill(L->dims);
    if (e != cudaSuccess) {
        delete L;
        return e == cudaErrorInvalidValue ? MOE_ERR_UNSUPPORTED : from_cuda(e);
    }
    const size_t max_groups = gemm ? qe::prefill_max_groups(L->dims, cfg->max_tokens) : 0;
    L->ws_bytes = carve(*cfg, max_groups, nullptr, nullptr, nullptr, nullptr);
    e = cudaMalloc(&L->ws_base, L->ws_bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        delete L;
        return MOE_ERR_OOM;
    }
    carve(*cfg, max_groups, (char*)L->ws_base, &L->ws, L->x_stage, &L->out_stage);
    e = cudaMemset(L->ws_base, 0, L->ws_bytes);
    if (e == cudaSuccess) {
        // the pointer table: expert e at its place in the contiguous [E] arrays
        const size_t E = (size_t)cfg->n_experts, f = (size_t)cfg->f, d = (size_t)cfg->d;
        const size_t gu_bytes = 2 * f * row_bytes(cfg->wkind, d), dn_bytes = d * row_bytes(cfg->wkind, f);
        std::vector<const void*> tab(4 * E);
        const bool scaled = cfg->wkind != MOE_W_BF16;
        for (size_t i = 0; i < E; ++i) {
            tab[i] = static_cast<const char*>(w->gate_up) + i * gu_bytes;
            tab[E + i] = scaled ? w->gate_up_scale + i * 2 * f : nullptr;
            tab[2 * E + i] = static_cast<const char*>(w->down) + i * dn_bytes;
            tab[3 * E + i] = scaled ? w->down_scale + i * d : nullptr;
        }
        e = cudaMemcpy(L->ws.etab, tab.data(), sizeof(void*) * 4 * E, cudaMemcpyHostToDevice);
    }
    if (e != cudaSuccess) {
        cudaFree(L->ws_base);
        delete L;
        return from_cuda(e);
    }
    if (gemm) {
        L->plan = qe::prefill_plan_create(L->dims, L->w, L->ws, cfg->max_tokens);
        if (!L->plan) {
            cudaFree(L->ws_base);
            delete L;
            return MOE_ERR_CUDA;
        }
    }
    // the host-buffer calls' copy stream and the events that order it with the caller's stream
    e = cudaStreamCreateWithFlags(&L->copy_s, cudaStreamNonBlocking);
    for (int i = 0; i < 2 && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&L->x_landed[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&L->x_read[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) {
        destroy_streams(L);
        qe::prefill_plan_destroy(L->plan);
        cudaFree(L->ws_base);
        delete L;
        return from_cuda(e);
    }
    L->t1_mode = L->fused_ok ? 2 : qe::decode_t1_supported(L->dims) ? 1 : 0;
    L->last_stream = nullptr;
    *out = L;
    return MOE_OK;
}

moe_status moe_route(moe_layer* L, const uint16_t* x, int32_t T, int32_t* idx, float* w, moe_stream stream) {
    if (!L || T < 0 || T > L->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !idx || !w || !aligned16(x) || ((uintptr_t)idx & 3) || ((uintptr_t)w & 3)) return MOE_ERR_INVALID_ARG;
    cudaGetLastError();   // an error left pending by an earlier, unrelated call is not this call's
    cudaStream_t s = (cudaStream_t)stream;
    int launches = 0;
    const qe::Launch ctx{s, &launches, &L->prof};
    cudaError_t e = qe::launch_router(L->dims, L->w.router_w, L->w.router_bias, x, T, L->ws.logits, L->ws.xsum, idx, w,
                                      nullptr, ctx, L->ws.rsplit, L->ws.rsplit_n);
    L->last_stream = s;
    L->last_launches = launches;
    return from_cuda(e);
}

moe_status moe_forward(moe_layer* L, const uint16_t* x, int32_t T, void* out, moe_stream stream) {
    if (!L || T < 0 || T > L->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x || !out || !aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
    cudaGetLastError();   // an error left pending by an earlier, unrelated call is not this call's
    cudaStream_t s = (cudaStream_t)stream;
    int launches = 0;
    const qe::Launch ctx{s, &launches, &L->prof};
    const qe::Workspace& ws = L->ws;
    const bool gemm = L->plan && !L->ragged && T >= L->prefill_min_tokens;
    cudaError_t e;
    // the single-token paths take the plain router only (a router variant may drop experts)
    const bool variant = L->dims.ropts.active();
    if (T <= 2 && L->t1_mode == 2 && !variant && (T == 1 || L->fused2_ok)) {
        e = qe::launch_decode_fused(L->dims, L->w, x, ws, out, L->num_sms, ctx, T);
        L->last_stream = s;
        L->last_launches = launches;
        return from_cuda(e);
    }
    if (T <= qe::kRouteSmallMaxT && qe::route_small_ok(L->dims, L->num_sms)) {
        e = qe::launch_route_small(L->dims, L->w.router_w, L->w.router_bias, x, T, ws, L->num_sms, ctx);
    } else {
        e = qe::launch_router(L->dims, L->w.router_w, L->w.router_bias, x, T, ws.logits, ws.xsum, ws.idx, ws.wts,
                              ws.asc, ctx, ws.rsplit, ws.rsplit_n);
        if (e == cudaSuccess) e = qe::launch_bucket(L->dims, T, ws, ctx);
    }
    if (e == cudaSuccess) {
        if (gemm) {
            e = qe::launch_prefill_experts(L->dims, L->plan, L->w, x, T, ws, L->num_sms, ctx);
            if (e == cudaSuccess) e = qe::launch_combine(L->dims, T, ws, out, ctx);
        } else if (T == 1 && L->t1_mode >= 1 && !variant) {
            e = qe::launch_decode_t1(L->dims, L->w, x, ws, out, L->num_sms, ctx);
        } else {
            e = L->union_mma && qe::decode_mma_ok(L->dims, T)
                    ? qe::launch_decode_mma(L->dims, L->w, x, T, ws, L->num_sms, ctx)
                    : qe::launch_decode_experts(L->dims, L->w, x, T, ws, L->num_sms, ctx);
            if (e == cudaSuccess) e = qe::launch_combine(L->dims, T, ws, out, ctx);
        }
    }
    L->last_stream = s;
    L->last_launches = launches;
    return from_cuda(e);
}

moe_status moe_layer_set_expert(moe_layer* L, int32_t e, const void* gate_up, const float* gate_up_scale,
                                const void* down, const float* down_scale, moe_stream stream) {
    if (!L || e < 0 || e >= L->cfg.n_experts || !gate_up || !down) return MOE_ERR_INVALID_ARG;
    const bool scaled = L->cfg.wkind != MOE_W_BF16;
    if (scaled && (!gate_up_scale || !down_scale)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(gate_up) || !aligned16(down) || (scaled && (!aligned16(gate_up_scale) || !aligned16(down_scale))))
        return MOE_ERR_INVALID_ARG;
    cudaGetLastError();
    cudaStream_t s = (cudaStream_t)stream;
    set_expert_kernel<<<1, 1, 0, s>>>(L->ws.etab, L->cfg.n_experts, e, gate_up, scaled ? gate_up_scale : nullptr, down,
                                      scaled ? down_scale : nullptr);
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return from_cuda(err);
    L->ragged = true;
    L->last_stream = s;
    return MOE_OK;
}

moe_status moe_forward_host_async(moe_layer* L, const uint16_t* x_host, int32_t T, void* out_host,
                                  moe_stream stream) {
    if (!L || T < 0 || T > L->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t xbytes = sizeof(uint16_t) * (size_t)T * L->cfg.d;
    const size_t obytes = (L->cfg.out_bf16 ? 2 : 4) * (size_t)T * L->cfg.d;
    // x goes in on the layer's copy stream into one of two stages, so that it can land while the
    // previous call's kernels still run; the stage is reused only once the kernels of the call
    // before that have read it
    const int i = L->x_next;
    L->x_next ^= 1;
    cudaError_t e = cudaStreamWaitEvent(L->copy_s, L->x_read[i], 0);
    if (e == cudaSuccess) e = cudaMemcpyAsync(L->x_stage[i], x_host, xbytes, cudaMemcpyHostToDevice, L->copy_s);
    if (e == cudaSuccess) e = cudaEventRecord(L->x_landed[i], L->copy_s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, L->x_landed[i], 0);
    if (e != cudaSuccess) return from_cuda(e);
    // A small output in mapped pinned host memory is written there by the kernels themselves (no
    // device -> host copy); anything else goes through the staging buffer and one copy.
    void* direct = nullptr;
    cudaPointerAttributes pa;
    if (obytes <= kDirectOutputBytes && cudaPointerGetAttributes(&pa, out_host) == cudaSuccess &&
        pa.type == cudaMemoryTypeHost && pa.devicePointer && aligned16(pa.devicePointer))
        direct = pa.devicePointer;
    cudaGetLastError();                 // a pointer the runtime does not know is not an error here
    moe_status st = moe_forward(L, L->x_stage[i], T, direct ? direct : L->out_stage, stream);
    if (st != MOE_OK) return st;
    e = cudaEventRecord(L->x_read[i], s);
    if (e == cudaSuccess && !direct) e = cudaMemcpyAsync(out_host, L->out_stage, obytes, cudaMemcpyDeviceToHost, s);
    return from_cuda(e);
}

moe_status moe_forward_host(moe_layer* L, const uint16_t* x_host, int32_t T, void* out_host, moe_stream stream) {
    const moe_status st = moe_forward_host_async(L, x_host, T, out_host, stream);
    if (st != MOE_OK || T == 0) return st;
    return from_cuda(cudaStreamSynchronize((cudaStream_t)stream));
}

moe_status moe_last_error(moe_layer* L) {
    if (!L) return MOE_ERR_INVALID_ARG;
    cudaError_t e = L->last_stream ? cudaStreamSynchronize(L->last_stream) : cudaDeviceSynchronize();
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    int st = 0;
    e = cudaMemcpy(&st, L->ws.status, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    if (st != 0) {
        e = cudaMemset(L->ws.status, 0, sizeof(int));
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    return (moe_status)st;
}

void moe_layer_destroy(moe_layer* L) {
    if (!L) return;
    if (L->last_stream) cudaStreamSynchronize(L->last_stream);
    else cudaDeviceSynchronize();
    if (L->copy_s) cudaStreamSynchronize(L->copy_s);
    destroy_streams(L);
    cudaFree(L->ws_base);
    qe::prefill_plan_destroy(L->plan);
    delete L;
}

moe_status moe_layer_set_option(moe_layer* L, int32_t option, int64_t value) {
    if (!L) return MOE_ERR_INVALID_ARG;
    switch (option) {
        case MOE_OPT_PREFILL_MIN_TOKENS:
            if (value < 1) return MOE_ERR_INVALID_ARG;
            L->prefill_min_tokens = value;
            return MOE_OK;
        case MOE_OPT_SINGLE_TOKEN_KERNELS: {
            if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
            int m = (int)value;
            if (m == 2 && !L->fused_ok) m = 1;
            if (m == 1 && !qe::decode_t1_supported(L->dims)) m = 0;
            L->t1_mode = m;
            return MOE_OK;
        }
        case MOE_OPT_PROGRAMMATIC_LAUNCH:
            if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
            L->dims.pdl = (int)value;
            return MOE_OK;
        case MOE_OPT_WAIT_LIMIT_US:
            if (value < 100 || value > 10000000) return MOE_ERR_INVALID_ARG;
            L->dims.wait_ns = (uint64_t)value * 1000ull;
            return MOE_OK;
        case MOE_OPT_TEST_SKIP_GEMM_B_COPIES:
            if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
            L->dims.test_skip_b = (int)value;
            return MOE_OK;
        case MOE_OPT_ROUTER_GROUPS: {
            const int G = (int)(value & 0xFFFF), TG = (int)(value >> 16);
            if (value < 0 || G < 1) return MOE_ERR_INVALID_ARG;
            if (G == 1) {
                L->dims.ropts.n_group = 1;
                L->dims.ropts.topk_group = 1;
                return MOE_OK;
            }
            const int E = L->cfg.n_experts;
            if (G > 32 || E % G || TG < 1 || TG > G || (int64_t)TG * (E / G) < L->cfg.top_k) return MOE_ERR_INVALID_ARG;
            L->dims.ropts.n_group = G;
            L->dims.ropts.topk_group = TG;
            return MOE_OK;
        }
        case MOE_OPT_ROUTER_TOP_P:
            if (value < 0 || value > 1000000) return MOE_ERR_INVALID_ARG;
            L->dims.ropts.top_p = (double)value * 1e-6;
            return MOE_OK;
        case MOE_OPT_UNION_TENSOR_CORES:
            if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
            L->union_mma = value != 0;
            return MOE_OK;
        case MOE_OPT_PHASE_TRACE:
            if (value != 0 && value != 1) return MOE_ERR_INVALID_ARG;
            L->dims.phase_trace = (int)value;
            return MOE_OK;
        default:
            return MOE_ERR_INVALID_ARG;
    }
}

moe_status moe_layer_debug_read(moe_layer* L, int32_t item, void* dst, int64_t bytes) {
    if (!L || !dst || bytes < 0) return MOE_ERR_INVALID_ARG;
    const size_t T = (size_t)L->cfg.max_tokens, k = (size_t)L->cfg.top_k, E = (size_t)L->cfg.n_experts;
    const size_t slots = T * k + T * (size_t)L->dims.S;
    const size_t fmax = L->dims.S && L->dims.f_shared > L->dims.f ? (size_t)L->dims.f_shared : (size_t)L->dims.f;
    const void* src = nullptr;
    size_t n = 0;
    switch (item) {
        case MOE_DEBUG_H: src = L->ws.h; n = 2 * slots * fmax; break;
        case MOE_DEBUG_Y: src = L->ws.Y; n = 4 * slots * (size_t)L->cfg.d; break;
        case MOE_DEBUG_IDX: src = L->ws.idx; n = 4 * T * k; break;
        case MOE_DEBUG_W: src = L->ws.wts; n = 4 * T * k; break;
        case MOE_DEBUG_ASC: src = L->ws.asc; n = 4 * T * k; break;
        case MOE_DEBUG_ULIST: src = L->ws.ulist; n = 4 * E; break;
        case MOE_DEBUG_CNT: src = L->ws.cnt; n = 4 * E; break;
        case MOE_DEBUG_XSUM: src = L->ws.xsum; n = 8 * T; break;
        case MOE_DEBUG_TRACE: src = L->ws.trace; n = 8 * (size_t)L->num_sms * qe::kTraceStamps; break;
        default: return MOE_ERR_INVALID_ARG;
    }
    if ((size_t)bytes < n) n = (size_t)bytes;
    cudaError_t e = L->last_stream ? cudaStreamSynchronize(L->last_stream) : cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(dst, src, n, cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status moe_layer_get_option(const moe_layer* L, int32_t option, int64_t* value) {
    if (!L || !value) return MOE_ERR_INVALID_ARG;
    switch (option) {
        case MOE_OPT_PREFILL_MIN_TOKENS: *value = L->prefill_min_tokens; return MOE_OK;
        case MOE_OPT_PREFILL_AVAILABLE: *value = L->plan && !L->ragged ? 1 : 0; return MOE_OK;
        case MOE_OPT_SINGLE_TOKEN_KERNELS: *value = L->t1_mode; return MOE_OK;
        case MOE_OPT_PROGRAMMATIC_LAUNCH: *value = L->dims.pdl; return MOE_OK;
        case MOE_OPT_WAIT_LIMIT_US: *value = (int64_t)(L->dims.wait_ns / 1000ull); return MOE_OK;
        case MOE_OPT_TEST_SKIP_GEMM_B_COPIES: *value = L->dims.test_skip_b; return MOE_OK;
        case MOE_OPT_ROUTER_GROUPS:
            *value = L->dims.ropts.n_group + ((int64_t)L->dims.ropts.topk_group << 16);
            return MOE_OK;
        case MOE_OPT_ROUTER_TOP_P: *value = (int64_t)(L->dims.ropts.top_p * 1e6 + 0.5); return MOE_OK;
        case MOE_OPT_UNION_TENSOR_CORES: *value = L->union_mma ? 1 : 0; return MOE_OK;
        case MOE_OPT_PHASE_TRACE: *value = L->dims.phase_trace; return MOE_OK;
        default: return MOE_ERR_INVALID_ARG;
    }
}

int64_t moe_layer_workspace_bytes(const moe_layer* L) { return L ? (int64_t)L->ws_bytes : 0; }

int32_t moe_layer_last_launches(const moe_layer* L) { return L ? L->last_launches : 0; }

moe_status moe_profile_enable(moe_layer* L, int32_t on) {
    if (!L) return MOE_ERR_INVALID_ARG;
    L->prof.on = on != 0;
    return MOE_OK;
}

moe_status moe_profile_read(moe_layer* L, int32_t kernel, double* total_ms, int64_t* launches) {
    if (!L || kernel < 0 || kernel >= MOE_KERNEL_COUNT || !total_ms || !launches) return MOE_ERR_INVALID_ARG;
    cudaError_t e = L->last_stream ? cudaStreamSynchronize(L->last_stream) : cudaDeviceSynchronize();
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    L->prof.collect();
    *total_ms = L->prof.total_ms[kernel];
    *launches = L->prof.count[kernel];
    L->prof.total_ms[kernel] = 0.0;
    L->prof.count[kernel] = 0;
    return MOE_OK;
}

const char* moe_kernel_name(int32_t kernel) {
    static const char* names[MOE_KERNEL_COUNT] = {"router_logits", "topk", "bucket", "gateup", "down", "combine",
                                                  "gather", "gemm_gateup", "gemm_down", "fused"};
    return (kernel >= 0 && kernel < MOE_KERNEL_COUNT) ? names[kernel] : "unknown";
}

}  // extern "C"
