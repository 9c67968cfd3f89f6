// cache.cu -- a device-memory tier of routed experts in front of host memory.
//
// The colibri README ("The idea") keeps the routed experts out of fast memory and streams each
// one on demand when a token routes to it, behind a per-layer LRU cache and an optional pinned
// hot set; the iliria page ("What's implemented") keeps them in pinned/LRU slabs behind a ragged
// descriptor.  Here HBM is the fast tier: n_slots expert-sized device buffers hold the experts
// in use, host memory holds all E of them, and the layer reads its experts through its pointer
// table (moe_layer_set_expert), so a routed expert can live in any slot.
//
// prepare(x): route the batch (the host needs the expert ids, so it waits for the routing), then
// for every expert the batch needs that no slot holds, take a free slot or evict the least
// recently used one that is neither pinned nor needed by this batch, copy the expert in
// (host -> device, one copy per array, on the caller's stream) and point the table at it.  The
// forward enqueued after it on the same stream sees the experts in place.
#include <cstring>
#include <new>
#include <vector>

#include "internal.cuh"

struct moe_expert_cache {
    moe_config cfg;
    moe_weights host;               // the routed experts in host memory
    moe_layer* layer = nullptr;
    void* slab = nullptr;           // n_slots x slot_bytes of device memory
    size_t gu_bytes = 0, gus_bytes = 0, dn_bytes = 0, dns_bytes = 0, slot_bytes = 0;
    int n_slots = 0;
    std::vector<int> slot_of;       // [E] slot holding expert e, or -1
    std::vector<int> expert_in;     // [n_slots] expert in slot s, or -1
    std::vector<int64_t> last_use;  // [n_slots] the prepare call that last needed it
    std::vector<char> pinned;       // [E]
    int64_t clock = 0, hits = 0, misses = 0, bytes_in = 0;
    int32_t* idx_dev = nullptr;     // [max_tokens][k] routing of the batch being prepared
    float* w_dev = nullptr;
    int32_t* idx_host = nullptr;    // pinned copy
};

namespace {

size_t row_bytes_of(int wkind, size_t cols) {
    switch (wkind) {
        case MOE_W_INT4_ROWSCALE: return cols / 2;
        case MOE_W_INT8_ROWSCALE: return cols;
        case MOE_W_INT2_ROWSCALE: return cols / 4;
        default: return cols * 2;
    }
}

moe_status status_of(cudaError_t e) {
    if (e == cudaSuccess) return MOE_OK;
    return e == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA;
}

char* slot_base(moe_expert_cache* c, int s) { return static_cast<char*>(c->slab) + (size_t)s * c->slot_bytes; }

// Points expert e at slot s (or, for s < 0, at slot 0: memory that is always valid to read).
moe_status point(moe_expert_cache* c, int e, int s, cudaStream_t st) {
    char* b = slot_base(c, s < 0 ? 0 : s);
    const bool scaled = c->cfg.wkind != MOE_W_BF16;
    return moe_layer_set_expert(c->layer, e, b, scaled ? reinterpret_cast<const float*>(b + c->gu_bytes) : nullptr,
                                b + c->gu_bytes + c->gus_bytes,
                                scaled ? reinterpret_cast<const float*>(b + c->gu_bytes + c->gus_bytes + c->dn_bytes)
                                       : nullptr,
                                (moe_stream)st);
}

void destroy(moe_expert_cache* c) {
    if (!c) return;
    if (c->layer) moe_layer_destroy(c->layer);
    cudaFree(c->slab);
    cudaFree(c->idx_dev);
    cudaFree(c->w_dev);
    cudaFreeHost(c->idx_host);
    delete c;
}

}  // namespace

extern "C" {

moe_status moe_expert_cache_create(const moe_config* cfg, const moe_weights* device, const moe_weights* host,
                                   int32_t n_slots, moe_expert_cache** out) {
    if (!cfg || !device || !host || !out || n_slots < 1) return MOE_ERR_INVALID_ARG;
    if (cfg->n_experts < 1 || n_slots > cfg->n_experts) return MOE_ERR_INVALID_ARG;
    const bool scaled = cfg->wkind != MOE_W_BF16;
    if (!host->gate_up || !host->down || (scaled && (!host->gate_up_scale || !host->down_scale)))
        return MOE_ERR_INVALID_ARG;
    moe_expert_cache* c = new (std::nothrow) moe_expert_cache();
    if (!c) return MOE_ERR_OOM;
    c->cfg = *cfg;
    c->host = *host;
    const size_t d = (size_t)cfg->d, f = (size_t)cfg->f;
    c->gu_bytes = 2 * f * row_bytes_of(cfg->wkind, d);
    c->gus_bytes = scaled ? 2 * f * sizeof(float) : 0;
    c->dn_bytes = d * row_bytes_of(cfg->wkind, f);
    c->dns_bytes = scaled ? d * sizeof(float) : 0;
    // every array of a slot starts on a 16-byte boundary (all four sizes are multiples of 16)
    c->slot_bytes = c->gu_bytes + c->gus_bytes + c->dn_bytes + c->dns_bytes;
    c->n_slots = n_slots;
    c->slot_of.assign((size_t)cfg->n_experts, -1);
    c->expert_in.assign((size_t)n_slots, -1);
    c->last_use.assign((size_t)n_slots, -1);
    c->pinned.assign((size_t)cfg->n_experts, 0);
    cudaError_t e = cudaMalloc(&c->slab, c->slot_bytes * (size_t)n_slots);
    if (e == cudaSuccess) e = cudaMemset(c->slab, 0, c->slot_bytes * (size_t)n_slots);
    const size_t tk = (size_t)cfg->max_tokens * (size_t)cfg->top_k;
    if (e == cudaSuccess) e = cudaMalloc((void**)&c->idx_dev, sizeof(int32_t) * tk);
    if (e == cudaSuccess) e = cudaMalloc((void**)&c->w_dev, sizeof(float) * tk);
    if (e == cudaSuccess) e = cudaMallocHost((void**)&c->idx_host, sizeof(int32_t) * tk);
    if (e != cudaSuccess) {
        cudaGetLastError();
        destroy(c);
        return status_of(e);
    }
    // the layer over slot 0 (its own contiguous-array view is never used: every expert is
    // pointed at a slot before the first forward)
    moe_weights w = *device;
    char* b = slot_base(c, 0);
    w.gate_up = b;
    w.gate_up_scale = scaled ? reinterpret_cast<const float*>(b + c->gu_bytes) : nullptr;
    w.down = b + c->gu_bytes + c->gus_bytes;
    w.down_scale = scaled ? reinterpret_cast<const float*>(b + c->gu_bytes + c->gus_bytes + c->dn_bytes) : nullptr;
    moe_config lc = *cfg;
    moe_status st = moe_layer_create(&lc, &w, &c->layer);
    if (st != MOE_OK) {
        c->layer = nullptr;
        destroy(c);
        return st;
    }
    for (int i = 0; i < cfg->n_experts && st == MOE_OK; ++i) st = point(c, i, -1, nullptr);
    if (st == MOE_OK) st = status_of(cudaDeviceSynchronize());
    if (st != MOE_OK) {
        destroy(c);
        return st;
    }
    *out = c;
    return MOE_OK;
}

moe_layer* moe_expert_cache_layer(moe_expert_cache* c) { return c ? c->layer : nullptr; }

moe_status moe_expert_cache_prepare(moe_expert_cache* c, const uint16_t* x, int32_t T, moe_stream stream) {
    if (!c || T < 0 || T > c->cfg.max_tokens) return MOE_ERR_INVALID_ARG;
    if (T == 0) return MOE_OK;
    cudaStream_t s = (cudaStream_t)stream;
    const int k = c->cfg.top_k, E = c->cfg.n_experts;
    moe_status st = moe_route(c->layer, x, T, c->idx_dev, c->w_dev, stream);
    if (st != MOE_OK) return st;
    cudaError_t e = cudaMemcpyAsync(c->idx_host, c->idx_dev, sizeof(int32_t) * (size_t)T * k, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // the batch's experts (index -1: dropped by adaptive top-p)
    std::vector<char> need((size_t)E, 0);
    std::vector<int> list;
    for (int i = 0; i < T * k; ++i) {
        const int ex = c->idx_host[i];
        if (ex >= 0 && ex < E && !need[(size_t)ex]) {
            need[(size_t)ex] = 1;
            list.push_back(ex);
        }
    }
    if ((int)list.size() > c->n_slots) return MOE_ERR_UNSUPPORTED;
    ++c->clock;
    for (int ex : list) {                          // the resident ones are hits; keep them
        const int sl = c->slot_of[(size_t)ex];
        if (sl >= 0) {
            ++c->hits;
            c->last_use[(size_t)sl] = c->clock;
        }
    }
    for (int ex : list) {
        if (c->slot_of[(size_t)ex] >= 0) continue;
        // a free slot, else the least recently used slot whose expert is neither pinned nor needed
        int best = -1;
        for (int sl = 0; sl < c->n_slots; ++sl) {
            const int held = c->expert_in[(size_t)sl];
            if (held < 0) { best = sl; break; }
            if (c->pinned[(size_t)held] || need[(size_t)held]) continue;
            if (best < 0 || c->last_use[(size_t)sl] < c->last_use[(size_t)best]) best = sl;
        }
        if (best < 0) return MOE_ERR_UNSUPPORTED;    // every slot is pinned or needed
        const int old = c->expert_in[(size_t)best];
        if (old >= 0) {
            c->slot_of[(size_t)old] = -1;
            if ((st = point(c, old, -1, s)) != MOE_OK) return st;
        }
        char* b = slot_base(c, best);
        const char* hg = static_cast<const char*>(c->host.gate_up) + (size_t)ex * c->gu_bytes;
        const char* hd = static_cast<const char*>(c->host.down) + (size_t)ex * c->dn_bytes;
        e = cudaMemcpyAsync(b, hg, c->gu_bytes, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess && c->gus_bytes)
            e = cudaMemcpyAsync(b + c->gu_bytes, reinterpret_cast<const char*>(c->host.gate_up_scale) + (size_t)ex * c->gus_bytes,
                                c->gus_bytes, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaMemcpyAsync(b + c->gu_bytes + c->gus_bytes, hd, c->dn_bytes, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess && c->dns_bytes)
            e = cudaMemcpyAsync(b + c->gu_bytes + c->gus_bytes + c->dn_bytes,
                                reinterpret_cast<const char*>(c->host.down_scale) + (size_t)ex * c->dns_bytes, c->dns_bytes,
                                cudaMemcpyHostToDevice, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
        if ((st = point(c, ex, best, s)) != MOE_OK) return st;
        c->expert_in[(size_t)best] = ex;
        c->slot_of[(size_t)ex] = best;
        c->last_use[(size_t)best] = c->clock;
        ++c->misses;
        c->bytes_in += (int64_t)c->slot_bytes;
    }
    return MOE_OK;
}

moe_status moe_expert_cache_pin(moe_expert_cache* c, int32_t e, int32_t pinned) {
    if (!c || e < 0 || e >= c->cfg.n_experts) return MOE_ERR_INVALID_ARG;
    c->pinned[(size_t)e] = pinned ? 1 : 0;
    return MOE_OK;
}

moe_status moe_expert_cache_stats(const moe_expert_cache* c, int64_t* hits, int64_t* misses, int64_t* bytes_in,
                                  int32_t* resident) {
    if (!c || !hits || !misses || !bytes_in || !resident) return MOE_ERR_INVALID_ARG;
    *hits = c->hits;
    *misses = c->misses;
    *bytes_in = c->bytes_in;
    int r = 0;
    for (int s = 0; s < c->n_slots; ++s) r += c->expert_in[(size_t)s] >= 0;
    *resident = r;
    return MOE_OK;
}

int32_t moe_expert_cache_slot_of(const moe_expert_cache* c, int32_t e) {
    if (!c || e < 0 || e >= c->cfg.n_experts) return -1;
    return c->slot_of[(size_t)e];
}

void moe_expert_cache_destroy(moe_expert_cache* c) {
    if (c && c->layer) moe_last_error(c->layer);       // waits for the layer's last stream
    destroy(c);
}

}  // extern "C"
