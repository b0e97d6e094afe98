// csa_api.cu -- the extern "C" boundary of libcsa_b200.so (see csa_b200.h).
//
// Every entry point validates its arguments on the host, maps them onto the
// internal launch structs and launches on the caller's stream.  Nothing is
// allocated, nothing is synchronised, no exception or abort crosses the ABI.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <cmath>

#include "csa_b200.h"
#include "kernels.h"

namespace csa {
static std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// One error word per device for kernels whose bounded waits expired.
static __device__ uint32_t g_device_error;
// Its device address per device, looked up once.  Host threads may race on
// the first lookup; they all store the same address, and the atomics make
// that race well defined.
static std::atomic<uint32_t*> g_error_ptr[64];

uint32_t* device_error_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    uint32_t* w = g_error_ptr[dev].load(std::memory_order_acquire);
    if (!w) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        w = static_cast<uint32_t*>(p);
        g_error_ptr[dev].store(w, std::memory_order_release);
    }
    return w;
}

// The wait limit the tensor-core kernels' work is launched with (ns).
static std::atomic<uint64_t> g_wait_limit_ns{1000000000ull};
static std::atomic<int> g_stall_next{0};
uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }
void set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns, std::memory_order_relaxed); }
int take_stall() { return g_stall_next.exchange(0); }
void set_stall(int on) { g_stall_next.store(on ? 1 : 0); }
}  // namespace csa

namespace {

thread_local char g_detail[512] = "";

csa_status_t fail(csa_status_t st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return st;
}

csa_status_t ok() {
    g_detail[0] = '\0';
    return CSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Test hook: an error the next launch returns instead of launching (one shot).
std::atomic<int> g_inject_error{0};

cudaError_t injected_or_launch_marker() {
    return static_cast<cudaError_t>(g_inject_error.exchange(0));
}

csa_status_t from_cuda(cudaError_t e, const char* what, const char* why) {
    if (e == cudaSuccess) return ok();
    if (e == cudaErrorNotSupported && why) return fail(CSA_ERR_UNSUPPORTED, "%s", why);
    return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define REQUIRE(cond, ...) \
    do {                   \
        if (!(cond)) return fail(CSA_ERR_INVALID_ARG, __VA_ARGS__); \
    } while (0)
// Every kernel launch of an entry point goes through LAUNCH: with an injected
// error pending (csa_debug_inject_launch_error) the launch is skipped and the
// error returned, as a failing launch would.
#define LAUNCH(expr) (g_inject_error.load() != 0 ? injected_or_launch_marker() : (expr))

#define REQUIRE_ALIGNED(p, name) \
    do {                         \
        if ((p) && !aligned16(p)) return fail(CSA_ERR_MISALIGNED, "%s is not 16-byte aligned", name); \
    } while (0)
// Per-element arrays (scales, weights, indices, positions, counts, LSE,
// block tables) are read and written one element at a time: 4-byte alignment.
#define REQUIRE_ALIGNED4(p, name) \
    do {                          \
        if ((p) && (reinterpret_cast<uintptr_t>(p) & 3u)) \
            return fail(CSA_ERR_MISALIGNED, "%s is not 4-byte aligned", name); \
    } while (0)

bool is_dt(int d) {
    return d == CSA_DT_F32 || d == CSA_DT_BF16 || d == CSA_DT_E4M3 || d == CSA_DT_E4M3_HADAMARD;
}
bool is_fp8(int d) { return d == CSA_DT_E4M3 || d == CSA_DT_E4M3_HADAMARD; }
bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }
// fp32(1/sqrt(d)), rounded as the oracle rounds it
float hadamard_norm(int d) { return (float)(1.0 / std::sqrt((double)d)); }

}  // namespace

extern "C" {

const char* csa_status_string(int status) {
    switch (status) {
        case CSA_OK: return "CSA_OK";
        case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
        case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
        case CSA_ERR_MISALIGNED: return "CSA_ERR_MISALIGNED";
        case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
        case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT";
    }
    return "CSA_ERR_UNKNOWN";
}

const char* csa_last_error_detail(void) { return g_detail; }

int csa_version(void) { return 100; }

unsigned long long csa_kernel_launches(void) { return csa::g_launches.load(); }

csa_status_t csa_check_device_error(void* stream, int clear) {
    uint32_t* p = csa::device_error_word();
    if (!p) return fail(CSA_ERR_CUDA, "csa_check_device_error: no device error word");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, p, sizeof v, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_check_device_error: %s", cudaGetErrorString(e));
    if (clear && v) {
        const uint32_t zero = 0;
        e = cudaMemcpyAsync(p, &zero, sizeof zero, cudaMemcpyHostToDevice, s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_check_device_error: %s", cudaGetErrorString(e));
    }
    if (v) return fail(CSA_ERR_TIMEOUT, "a device-side wait exceeded its time limit (code %u)", v);
    return ok();
}

csa_status_t csa_compress(const void* x, int x_dt, int B, int n, int d_in, const void* W,
                          int d_out, int m, int overlap, void* out, int out_dt,
                          float* out_row_scale, void* stream) {
    REQUIRE(B >= 0 && n >= 0, "csa_compress: negative B or n");
    REQUIRE(m >= 1, "csa_compress: m must be >= 1");
    REQUIRE(overlap == 0 || overlap == 1, "csa_compress: overlap must be 0 or 1");
    REQUIRE(is_dt(x_dt) && is_dt(out_dt), "csa_compress: unknown dtype");
    REQUIRE(d_in > 0 && d_out > 0, "csa_compress: d_in and d_out must be positive");
    if (d_in % 16 || d_out % 16 || d_in > 256 || d_out > 256)
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress: d_in, d_out must be multiples of 16 in [16, 256]");
    if (is_fp8(x_dt)) return fail(CSA_ERR_UNSUPPORTED, "csa_compress: fp8 input is not supported");
    if (out_dt == CSA_DT_E4M3_HADAMARD && !pow2(d_out))
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress: the Hadamard fp8 type needs d_out a power of two");
    if (out_dt == CSA_DT_F32 && x_dt != CSA_DT_F32)
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress: F32 output needs F32 input");
    const int N_c = n / m;
    REQUIRE((long)B * N_c == 0 || is_fp8(out_dt) == (out_row_scale != nullptr),
            "csa_compress: out_row_scale is required for E4M3 output and must be NULL otherwise");
    if ((long)B * N_c == 0) return ok();
    REQUIRE(x && W && out, "csa_compress: null tensor pointer");
    REQUIRE_ALIGNED(x, "x");
    REQUIRE_ALIGNED(W, "W");
    REQUIRE_ALIGNED(out, "out");
    REQUIRE_ALIGNED4(out_row_scale, "out_row_scale");
    csa::CompressArgs a{x, x_dt, B, n, d_in, W, d_out, m, overlap, out, out_dt, out_row_scale, N_c,
                        hadamard_norm(d_out)};
    const char* why = nullptr;
    return from_cuda(LAUNCH(csa::launch_compress(a, static_cast<cudaStream_t>(stream), &why)), "csa_compress", why);
}

csa_status_t csa_compress_gated(const void* x, int x_dt, int B, int n, int d_in, const void* W_kv,
                                const void* W_gate, const float* ape, int d_out, int m, int overlap,
                                void* out, int out_dt, float* out_row_scale, void* stream) {
    REQUIRE(B >= 0 && n >= 0, "csa_compress_gated: negative B or n");
    REQUIRE(m >= 1, "csa_compress_gated: m must be >= 1");
    REQUIRE(overlap == 0 || overlap == 1, "csa_compress_gated: overlap must be 0 or 1");
    REQUIRE(is_dt(x_dt) && is_dt(out_dt), "csa_compress_gated: unknown dtype");
    REQUIRE(d_in > 0 && d_out > 0, "csa_compress_gated: d_in and d_out must be positive");
    if (d_in % 16 || d_out % 16 || d_in > 256 || d_out > 256)
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress_gated: d_in, d_out must be multiples of 16 in [16, 256]");
    if (is_fp8(x_dt)) return fail(CSA_ERR_UNSUPPORTED, "csa_compress_gated: fp8 input is not supported");
    if (out_dt == CSA_DT_E4M3_HADAMARD && !pow2(d_out))
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress_gated: the Hadamard fp8 type needs d_out a power of two");
    if (out_dt == CSA_DT_F32 && x_dt != CSA_DT_F32)
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress_gated: F32 output needs F32 input");
    const int N_c = n / m;
    REQUIRE((long)B * N_c == 0 || is_fp8(out_dt) == (out_row_scale != nullptr),
            "csa_compress_gated: out_row_scale is required for E4M3 output and must be NULL otherwise");
    if ((long)B * N_c == 0) return ok();
    REQUIRE(x && W_kv && W_gate && ape && out, "csa_compress_gated: null tensor pointer");
    REQUIRE_ALIGNED(x, "x");
    REQUIRE_ALIGNED(W_kv, "W_kv");
    REQUIRE_ALIGNED(W_gate, "W_gate");
    REQUIRE_ALIGNED4(ape, "ape");
    REQUIRE_ALIGNED(out, "out");
    REQUIRE_ALIGNED4(out_row_scale, "out_row_scale");
    csa::GatedArgs a{x, x_dt, B, n, d_in, W_kv, W_gate, ape, d_out, m, overlap, out, out_dt,
                     out_row_scale, N_c, hadamard_norm(d_out)};
    const char* why = nullptr;
    return from_cuda(LAUNCH(csa::launch_compress_gated(a, static_cast<cudaStream_t>(stream), &why)),
                     "csa_compress_gated", why);
}

static csa_status_t compress_append_impl(const void* x_new, int x_dt, int B, int d_in, const void* W,
                                         int d_out, int m, int overlap, const int* pos, float* state,
                                         void* cache, int out_dt, float* cache_scale, int N_cap,
                                         int* n_entries, const csa::PageMap& pm, void* stream) {
    REQUIRE(B >= 0 && N_cap >= 0, "csa_compress_append: negative B or N_cap");
    REQUIRE(m >= 1, "csa_compress_append: m must be >= 1");
    REQUIRE(overlap == 0 || overlap == 1, "csa_compress_append: overlap must be 0 or 1");
    REQUIRE(is_dt(x_dt) && is_dt(out_dt), "csa_compress_append: unknown dtype");
    REQUIRE(d_in > 0 && d_out > 0, "csa_compress_append: d_in and d_out must be positive");
    if (d_in % 16 || d_out % 16 || d_in > 256 || d_out > 256)
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress_append: d_in, d_out must be multiples of 16 in [16, 256]");
    if (is_fp8(x_dt)) return fail(CSA_ERR_UNSUPPORTED, "csa_compress_append: fp8 input is not supported");
    if (out_dt == CSA_DT_E4M3_HADAMARD && !pow2(d_out))
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress_append: the Hadamard fp8 type needs d_out a power of two");
    if (out_dt == CSA_DT_F32 && x_dt != CSA_DT_F32)
        return fail(CSA_ERR_UNSUPPORTED, "csa_compress_append: F32 output needs F32 input");
    REQUIRE((long)B * N_cap == 0 || is_fp8(out_dt) == (cache_scale != nullptr),
            "csa_compress_append: cache_scale is required for E4M3 output and must be NULL otherwise");
    if (B == 0) return ok();
    REQUIRE(x_new && W && pos && state, "csa_compress_append: null pointer");
    REQUIRE(cache || N_cap == 0, "csa_compress_append: null cache");
    REQUIRE_ALIGNED(x_new, "x_new");
    REQUIRE_ALIGNED(W, "W");
    REQUIRE_ALIGNED4(state, "state");
    REQUIRE_ALIGNED(cache, "cache");
    REQUIRE_ALIGNED4(cache_scale, "cache_scale");
    csa::AppendArgs a{x_new, x_dt, B, d_in, W, d_out, m, overlap, pos, state, cache, out_dt,
                      cache_scale, N_cap, n_entries, hadamard_norm(d_out), pm};
    const char* why = nullptr;
    return from_cuda(LAUNCH(csa::launch_compress_append(a, static_cast<cudaStream_t>(stream), &why)),
                     "csa_compress_append", why);
}

static csa_status_t indexer_impl(const void* qI, int qI_dt, const float* qI_scale,
                                 const float* qI_weight, const void* kI, int kI_dt,
                                 const float* kI_scale, int B, int n_q, int H_I, int d_I, int N_cap,
                                 const int* n_entries, const int* q_pos, int m, int topk,
                                 int* idx_out, const csa::PageMap& pm, void* stream,
                                 int q_pos0 = 0) {
    REQUIRE(B >= 0 && n_q >= 0 && N_cap >= 0, "csa_indexer_topk: negative size");
    REQUIRE(q_pos0 >= 0, "csa_indexer_topk_at: q_pos0 must be >= 0");
    REQUIRE(H_I >= 1 && d_I >= 1, "csa_indexer_topk: H_I and d_I must be positive");
    REQUIRE(m >= 1, "csa_indexer_topk: m must be >= 1");
    REQUIRE(topk >= 1 && topk <= 2048, "csa_indexer_topk: topk must be in [1, 2048]");
    REQUIRE(is_dt(qI_dt) && is_dt(kI_dt), "csa_indexer_topk: unknown dtype");
    if (d_I % 16) return fail(CSA_ERR_UNSUPPORTED, "csa_indexer_topk: d_I must be a multiple of 16");
    if (qI_dt == CSA_DT_E4M3_HADAMARD)
        return fail(CSA_ERR_UNSUPPORTED, "csa_indexer_topk: give rotated query codes as CSA_DT_E4M3");
    REQUIRE((long)B * n_q == 0 || (qI_dt == CSA_DT_E4M3) == (qI_scale != nullptr),
            "csa_indexer_topk: qI_scale is required iff qI is E4M3");
    REQUIRE((long)B * N_cap == 0 || is_fp8(kI_dt) == (kI_scale != nullptr),
            "csa_indexer_topk: kI_scale is required iff kI is E4M3");
    if (kI_dt == CSA_DT_E4M3_HADAMARD && !pow2(d_I))
        return fail(CSA_ERR_UNSUPPORTED, "csa_indexer_topk: Hadamard keys need d_I a power of two");
    if ((long)B * n_q == 0) return ok();
    REQUIRE(qI && idx_out, "csa_indexer_topk: null tensor pointer");
    REQUIRE(kI || N_cap == 0, "csa_indexer_topk: null kI");
    REQUIRE_ALIGNED(qI, "qI");
    REQUIRE_ALIGNED(kI, "kI");
    REQUIRE_ALIGNED4(idx_out, "idx_out");
    REQUIRE_ALIGNED4(qI_scale, "qI_scale");
    REQUIRE_ALIGNED4(qI_weight, "qI_weight");
    REQUIRE_ALIGNED4(kI_scale, "kI_scale");
    REQUIRE_ALIGNED4(n_entries, "n_entries");
    REQUIRE_ALIGNED4(q_pos, "q_pos");
    csa::IndexerArgs a{qI, qI_dt, qI_scale, kI, kI_dt, kI_scale, B, n_q, H_I, d_I, N_cap,
                       n_entries, q_pos, m, topk, idx_out, hadamard_norm(d_I), qI_weight, pm};
    a.pos0 = q_pos0;
    const char* why = nullptr;
    return from_cuda(LAUNCH(csa::launch_indexer_topk(a, static_cast<cudaStream_t>(stream), &why)),
                     "csa_indexer_topk", why);
}

// The page map of a paged entry point (validated), or an error status.
static csa_status_t page_map(const char* name, int B, const int* block_table, int max_pages,
                             int page_size, int num_pages, csa::PageMap* pm, int* N_cap) {
    REQUIRE(max_pages >= 0 && num_pages >= 0, "%s: negative max_pages or num_pages", name);
    REQUIRE(page_size >= 1 && page_size <= (1 << 20) && pow2(page_size),
            "%s: page_size must be a power of two in [1, 2^20]", name);
    REQUIRE((long)max_pages * page_size <= (1L << 30), "%s: max_pages * page_size above 2^30", name);
    REQUIRE((long)num_pages * page_size <= (1L << 31) - 1, "%s: page pool above 2^31 - 1 rows", name);
    REQUIRE(block_table || B == 0 || max_pages == 0, "%s: null block_table", name);
    REQUIRE_ALIGNED4(block_table, "block_table");
    int shift = 0;
    while ((1 << shift) < page_size) ++shift;
    pm->bt = block_table;
    pm->max_pages = max_pages;
    pm->page_shift = shift;
    pm->num_pages = num_pages;
    *N_cap = max_pages * page_size;
    return ok();
}

csa_status_t csa_compress_append(const void* x_new, int x_dt, int B, int d_in, const void* W,
                                 int d_out, int m, int overlap, const int* pos, float* state,
                                 void* cache, int out_dt, float* cache_scale, int N_cap,
                                 int* n_entries, void* stream) {
    return compress_append_impl(x_new, x_dt, B, d_in, W, d_out, m, overlap, pos, state, cache,
                                out_dt, cache_scale, N_cap, n_entries, csa::PageMap{}, stream);
}

csa_status_t csa_compress_append_paged(const void* x_new, int x_dt, int B, int d_in, const void* W,
                                       int d_out, int m, int overlap, const int* pos, float* state,
                                       void* cache_pages, int out_dt, float* cache_scale_pages,
                                       const int* block_table, int max_pages, int page_size,
                                       int num_pages, int* n_entries, void* stream) {
    csa::PageMap pm;
    int N_cap = 0;
    const csa_status_t st = page_map("csa_compress_append_paged", B, block_table, max_pages,
                                     page_size, num_pages, &pm, &N_cap);
    if (st != CSA_OK) return st;
    return compress_append_impl(x_new, x_dt, B, d_in, W, d_out, m, overlap, pos, state,
                                cache_pages, out_dt, cache_scale_pages, N_cap, n_entries, pm,
                                stream);
}

csa_status_t csa_indexer_topk(const void* qI, int qI_dt, const float* qI_scale,
                              const float* qI_weight, const void* kI, int kI_dt,
                              const float* kI_scale, int B, int n_q, int H_I, int d_I, int N_cap,
                              const int* n_entries, const int* q_pos, int m, int topk,
                              int* idx_out, void* stream) {
    return indexer_impl(qI, qI_dt, qI_scale, qI_weight, kI, kI_dt, kI_scale, B, n_q, H_I, d_I,
                        N_cap, n_entries, q_pos, m, topk, idx_out, csa::PageMap{}, stream);
}

csa_status_t csa_indexer_topk_paged(const void* qI, int qI_dt, const float* qI_scale,
                                    const float* qI_weight, const void* kI_pages, int kI_dt,
                                    const float* kI_scale_pages, const int* block_table,
                                    int max_pages, int page_size, int num_pages, int B, int n_q,
                                    int H_I, int d_I, const int* n_entries, const int* q_pos,
                                    int m, int topk, int* idx_out, void* stream) {
    csa::PageMap pm;
    int N_cap = 0;
    const csa_status_t st = page_map("csa_indexer_topk_paged", B, block_table, max_pages,
                                     page_size, num_pages, &pm, &N_cap);
    if (st != CSA_OK) return st;
    return indexer_impl(qI, qI_dt, qI_scale, qI_weight, kI_pages, kI_dt, kI_scale_pages, B, n_q,
                        H_I, d_I, N_cap, n_entries, q_pos, m, topk, idx_out, pm, stream);
}

static csa_status_t attention_common(const char* name, csa::AttnArgs& a, void* stream) {
    REQUIRE(a.B >= 0 && a.n_q >= 0 && a.N_cap >= 0 && a.L_raw >= 0, "%s: negative size", name);
    REQUIRE(a.H >= 1 && a.D >= 1, "%s: H and D must be positive", name);
    REQUIRE(a.window >= 0, "%s: window must be >= 0", name);
    REQUIRE(is_dt(a.dt), "%s: unknown dtype", name);
    if (is_fp8(a.dt)) return fail(CSA_ERR_UNSUPPORTED, "%s: dt must be F32 or BF16", name);
    if (a.D % 16 || a.D > 256) return fail(CSA_ERR_UNSUPPORTED, "%s: D must be a multiple of 16 <= 256", name);
    if ((long)a.B * a.n_q == 0) return ok();
    REQUIRE(a.q && a.out, "%s: null q or out", name);
    REQUIRE(a.kv_c || a.N_cap == 0, "%s: null kv_c", name);
    REQUIRE(a.kv_raw || a.L_raw == 0, "%s: null kv_raw", name);
    REQUIRE_ALIGNED(a.q, "q");
    REQUIRE_ALIGNED(a.kv_c, "kv_c");
    REQUIRE_ALIGNED(a.kv_raw, "kv_raw");
    REQUIRE_ALIGNED(a.out, "out");
    REQUIRE_ALIGNED4(a.lse_out, "lse_out");
    REQUIRE_ALIGNED4(a.idx, "idx");
    REQUIRE_ALIGNED4(a.raw_pos0, "raw_pos0");
    REQUIRE_ALIGNED4(a.raw_len, "raw_len");
    REQUIRE_ALIGNED4(a.q_pos, "q_pos");
    REQUIRE_ALIGNED4(a.n_entries, "n_entries");
    if (!(a.scale > 0.0f)) a.scale = 1.0f / sqrtf((float)a.D);
    const char* why = nullptr;
    return from_cuda(LAUNCH(csa::launch_attention(a, static_cast<cudaStream_t>(stream), &why)), name, why);
}

csa_status_t csa_sparse_attn(const void* q, int dt, int B, int n_q, int H, int D,
                             const void* kv_c, int N_cap, const int* idx, int topk,
                             const void* kv_raw, int L_raw, const int* raw_pos0,
                             const int* raw_len, int window, const int* q_pos,
                             float softmax_scale, void* out, float* lse_out, void* stream) {
    REQUIRE(topk >= 0 && topk <= 2048, "csa_sparse_attn: topk must be in [0, 2048]");
    REQUIRE(idx || topk == 0 || (long)B * n_q == 0, "csa_sparse_attn: null idx");
    csa::AttnArgs a{q, dt, B, n_q, H, D, kv_c, N_cap, idx, topk, nullptr, 1, 0, kv_raw, L_raw,
                    raw_pos0, raw_len, window, q_pos, softmax_scale, out, lse_out};
    return attention_common("csa_sparse_attn", a, stream);
}

csa_status_t csa_sparse_attn_paged(const void* q, int dt, int B, int n_q, int H, int D,
                                   const void* kv_c_pages, const int* block_table, int max_pages,
                                   int page_size, int num_pages, const int* idx, int topk,
                                   const void* kv_raw, int L_raw, const int* raw_pos0,
                                   const int* raw_len, int window, const int* q_pos,
                                   float softmax_scale, void* out, float* lse_out, void* stream) {
    REQUIRE(topk >= 0 && topk <= 2048, "csa_sparse_attn_paged: topk must be in [0, 2048]");
    REQUIRE(idx || topk == 0 || (long)B * n_q == 0, "csa_sparse_attn_paged: null idx");
    csa::PageMap pm;
    int N_cap = 0;
    const csa_status_t st = page_map("csa_sparse_attn_paged", B, block_table, max_pages, page_size,
                                     num_pages, &pm, &N_cap);
    if (st != CSA_OK) return st;
    csa::AttnArgs a{q, dt, B, n_q, H, D, kv_c_pages, N_cap, idx, topk, nullptr, 1, 0, kv_raw,
                    L_raw, raw_pos0, raw_len, window, q_pos, softmax_scale, out, lse_out, pm};
    return attention_common("csa_sparse_attn_paged", a, stream);
}

csa_status_t hca_dense_attn(const void* q, int dt, int B, int n_q, int H, int D,
                            const void* kv_c, int N_cap, const int* n_entries, int m,
                            const void* kv_raw, int L_raw, const int* raw_pos0,
                            const int* raw_len, int window, const int* q_pos,
                            float softmax_scale, void* out, float* lse_out, void* stream) {
    REQUIRE(m >= 1, "hca_dense_attn: m must be >= 1");
    csa::AttnArgs a{q, dt, B, n_q, H, D, kv_c, N_cap, nullptr, 0, n_entries, m, 1, kv_raw, L_raw,
                    raw_pos0, raw_len, window, q_pos, softmax_scale, out, lse_out};
    return attention_common("hca_dense_attn", a, stream);
}

csa_status_t hca_dense_attn_paged(const void* q, int dt, int B, int n_q, int H, int D,
                                  const void* kv_c_pages, const int* block_table, int max_pages,
                                  int page_size, int num_pages, const int* n_entries, int m,
                                  const void* kv_raw, int L_raw, const int* raw_pos0,
                                  const int* raw_len, int window, const int* q_pos,
                                  float softmax_scale, void* out, float* lse_out, void* stream) {
    REQUIRE(m >= 1, "hca_dense_attn_paged: m must be >= 1");
    csa::PageMap pm;
    int N_cap = 0;
    const csa_status_t st = page_map("hca_dense_attn_paged", B, block_table, max_pages, page_size,
                                     num_pages, &pm, &N_cap);
    if (st != CSA_OK) return st;
    csa::AttnArgs a{q, dt, B, n_q, H, D, kv_c_pages, N_cap, nullptr, 0, n_entries, m, 1, kv_raw,
                    L_raw, raw_pos0, raw_len, window, q_pos, softmax_scale, out, lse_out, pm};
    return attention_common("hca_dense_attn_paged", a, stream);
}

// ------------------------------------------------------------ spans at an offset
csa_status_t csa_indexer_topk_at(const void* qI, int qI_dt, const float* qI_scale,
                                 const float* qI_weight, const void* kI, int kI_dt,
                                 const float* kI_scale, int B, int n_q, int H_I, int d_I,
                                 int N_cap, const int* n_entries, int q_pos0, int m, int topk,
                                 int* idx_out, void* stream) {
    return indexer_impl(qI, qI_dt, qI_scale, qI_weight, kI, kI_dt, kI_scale, B, n_q, H_I, d_I,
                        N_cap, n_entries, nullptr, m, topk, idx_out, csa::PageMap{}, stream,
                        q_pos0);
}

csa_status_t csa_sparse_attn_at(const void* q, int dt, int B, int n_q, int H, int D,
                                const void* kv_c, int N_cap, const int* idx, int topk,
                                const void* kv_raw, int L_raw, int raw_pos0, int window,
                                int q_pos0, float softmax_scale, void* out, float* lse_out,
                                void* stream) {
    REQUIRE(topk >= 0 && topk <= 2048, "csa_sparse_attn_at: topk must be in [0, 2048]");
    REQUIRE(idx || topk == 0 || (long)B * n_q == 0, "csa_sparse_attn_at: null idx");
    REQUIRE(q_pos0 >= 0 && raw_pos0 >= 0, "csa_sparse_attn_at: q_pos0 and raw_pos0 must be >= 0");
    csa::AttnArgs a{q, dt, B, n_q, H, D, kv_c, N_cap, idx, topk, nullptr, 1, 0, kv_raw, L_raw,
                    nullptr, nullptr, window, nullptr, softmax_scale, out, lse_out};
    a.pos0 = q_pos0;
    a.raw_base = raw_pos0;
    return attention_common("csa_sparse_attn_at", a, stream);
}

csa_status_t hca_dense_attn_at(const void* q, int dt, int B, int n_q, int H, int D,
                               const void* kv_c, int N_cap, const int* n_entries, int m,
                               const void* kv_raw, int L_raw, int raw_pos0, int window,
                               int q_pos0, float softmax_scale, void* out, float* lse_out,
                               void* stream) {
    REQUIRE(m >= 1, "hca_dense_attn_at: m must be >= 1");
    REQUIRE(q_pos0 >= 0 && raw_pos0 >= 0, "hca_dense_attn_at: q_pos0 and raw_pos0 must be >= 0");
    csa::AttnArgs a{q, dt, B, n_q, H, D, kv_c, N_cap, nullptr, 0, n_entries, m, 1, kv_raw, L_raw,
                    nullptr, nullptr, window, nullptr, softmax_scale, out, lse_out};
    a.pos0 = q_pos0;
    a.raw_base = raw_pos0;
    return attention_common("hca_dense_attn_at", a, stream);
}

// ------------------------------------------------------------------ test hooks
csa_status_t csa_debug_inject_launch_error(int cuda_error) {
    REQUIRE(cuda_error > 0, "csa_debug_inject_launch_error: the code must be a CUDA error (> 0)");
    // the packed entry points read cudaErrorNotSupported from a launch as
    // "take the per-sequence path", which would swallow the injected failure
    REQUIRE(cuda_error != (int)cudaErrorNotSupported,
            "csa_debug_inject_launch_error: cudaErrorNotSupported (801) is not a launch failure");
    g_inject_error.store(cuda_error);
    return ok();
}

csa_status_t csa_debug_set_wait_limit(long long ns, int stall_next) {
    REQUIRE(ns >= 0, "csa_debug_set_wait_limit: the limit must be >= 0 (0: the default 1 s)");
    csa::set_wait_limit_ns(ns == 0 ? 1000000000ull : (uint64_t)ns);
    csa::set_stall(stall_next);
    return ok();
}

// ------------------------------------------------------------------ varlen
// Packed sequences: sequence s owns tokens [cu[s], cu[s+1]) of the packed
// token dimension and entries [e(s), e(s+1)) of the packed compressed
// dimension, e(s) = sum over earlier sequences of floor(len/m).  Each call
// validates every sequence first, then launches the per-sequence kernels on
// the stream, so nothing is launched on a validation error.

static size_t dt_bytes(int dt) { return dt == CSA_DT_F32 ? 4 : (dt == CSA_DT_BF16 ? 2 : 1); }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

static csa_status_t check_cu(const char* name, int S, const int* cu, int m) {
    REQUIRE(S >= 0, "%s: negative S", name);
    REQUIRE(m >= 1, "%s: m must be >= 1", name);
    REQUIRE(cu || S == 0, "%s: null cu_seqlens", name);
    if (S == 0) return ok();
    REQUIRE(cu[0] == 0, "%s: cu_seqlens[0] must be 0", name);
    for (int s = 0; s < S; ++s)
        REQUIRE(cu[s + 1] >= cu[s], "%s: cu_seqlens must be non-decreasing (at %d)", name, s);
    return ok();
}

int csa_varlen_entry_offsets(const int* cu_seqlens, int S, int m, int* entry_offsets) {
    if (S < 0 || m < 1 || !entry_offsets || (S > 0 && !cu_seqlens)) return -1;
    if (S > 0 && cu_seqlens[0] != 0) return -1;
    for (int s = 0; s < S; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    long e = 0;
    entry_offsets[0] = 0;
    for (int s = 0; s < S; ++s) {
        e += (cu_seqlens[s + 1] - cu_seqlens[s]) / m;
        if (e > 0x7fffffffL) return -1;
        entry_offsets[s + 1] = (int)e;
    }
    return (int)e;
}

#define PTR_AT(p, elems, bytes) \
    ((p) ? static_cast<const void*>(static_cast<const uint8_t*>(p) + (size_t)(elems) * (bytes)) : nullptr)
#define MPTR_AT(p, elems, bytes) \
    ((p) ? static_cast<void*>(static_cast<uint8_t*>(p) + (size_t)(elems) * (bytes)) : nullptr)

csa_status_t csa_compress_varlen(const void* x, int x_dt, int S, const int* cu_seqlens, int d_in,
                                 const void* W, int d_out, int m, int overlap, void* out,
                                 int out_dt, float* out_row_scale, void* stream) {
    const char* name = "csa_compress_varlen";
    csa_status_t st = check_cu(name, S, cu_seqlens, m);
    if (st != CSA_OK) return st;
    REQUIRE(is_dt(x_dt) && is_dt(out_dt), "%s: unknown dtype", name);
    const long T = S > 0 ? cu_seqlens[S] : 0;
    // the shared arguments, once (a call with no batch launches nothing)
    st = csa_compress(x, x_dt, 0, 0, d_in, W, d_out, m, overlap, out, out_dt, out_row_scale, stream);
    if (st != CSA_OK) return st;
    REQUIRE(T == 0 || (x && W && out), "%s: null tensor pointer", name);
    long E = 0;
    for (int s = 0; s < S; ++s) E += (cu_seqlens[s + 1] - cu_seqlens[s]) / m;
    REQUIRE(E == 0 || is_fp8(out_dt) == (out_row_scale != nullptr),
            "%s: out_row_scale is required for E4M3 output and must be NULL otherwise", name);
    for (int pass = 0; pass < 2; ++pass) {          // pass 0 validates, pass 1 launches
        if (pass == 1 && S <= csa::kMaxVarlenSeqs) {   // one launch, offsets by value
            csa::VarlenMap map;
            map.S = S;
            int max_nc = 0;
            for (int s = 0; s <= S; ++s) {
                map.tok[s] = cu_seqlens[s];
                map.ent[s] = s == 0 ? 0 : map.ent[s - 1] + (cu_seqlens[s] - cu_seqlens[s - 1]) / m;
                if (s > 0) max_nc = std::max(max_nc, (cu_seqlens[s] - cu_seqlens[s - 1]) / m);
            }
            if (max_nc == 0) return ok();
            int max_len = 0;
            for (int s = 0; s < S; ++s) max_len = std::max(max_len, cu_seqlens[s + 1] - cu_seqlens[s]);
            csa::CompressArgs a{x, x_dt, S, max_len, d_in, W, d_out, m, overlap, out, out_dt,
                                out_row_scale, max_nc, hadamard_norm(d_out), &map};
            const char* why = nullptr;
            return from_cuda(LAUNCH(csa::launch_compress(a, static_cast<cudaStream_t>(stream), &why)), name,
                             why);
        }
        long e = 0;
        for (int s = 0; s < S; ++s) {
            const int L = cu_seqlens[s + 1] - cu_seqlens[s];
            const void* xs = PTR_AT(x, (long)cu_seqlens[s] * d_in, dt_bytes(x_dt));
            void* os = MPTR_AT(out, e * d_out, dt_bytes(out_dt));
            float* ss = out_row_scale ? out_row_scale + e : nullptr;
            if (L / m == 0) continue;
            if (pass == 0) {
                if (!(aligned16(xs) && aligned16(os) && (!ss || aligned4(ss))))
                    return fail(CSA_ERR_MISALIGNED, "%s: sequence %d's rows are not 16-byte aligned "
                                "(token offset %d)", name, s, cu_seqlens[s]);
            } else {
                st = csa_compress(xs, x_dt, 1, L, d_in, W, d_out, m, overlap, os, out_dt, ss, stream);
                if (st != CSA_OK) return st;
            }
            e += L / m;
        }
    }
    return ok();
}

csa_status_t csa_indexer_topk_varlen(const void* qI, int qI_dt, const float* qI_scale,
                                     const float* qI_weight, const void* kI, int kI_dt,
                                     const float* kI_scale, int S, const int* cu_seqlens, int H_I,
                                     int d_I, int m, int topk, int* idx_out, void* stream) {
    const char* name = "csa_indexer_topk_varlen";
    csa_status_t st = check_cu(name, S, cu_seqlens, m);
    if (st != CSA_OK) return st;
    REQUIRE(is_dt(qI_dt) && is_dt(kI_dt), "%s: unknown dtype", name);
    st = csa_indexer_topk(qI, qI_dt, qI_scale, qI_weight, kI, kI_dt, kI_scale, 0, 0, H_I, d_I, 0,
                          nullptr, nullptr, m, topk, idx_out, stream);
    if (st != CSA_OK) return st;
    REQUIRE(S == 0 || cu_seqlens[S] == 0 || (qI && idx_out), "%s: null tensor pointer", name);
    {
        long E = 0;
        for (int s = 0; s < S; ++s) E += (cu_seqlens[s + 1] - cu_seqlens[s]) / m;
        const long T = S > 0 ? cu_seqlens[S] : 0;
        REQUIRE(E == 0 || kI, "%s: null kI", name);
        REQUIRE(T == 0 || (qI_dt == CSA_DT_E4M3) == (qI_scale != nullptr),
                "%s: qI_scale is required iff qI is E4M3", name);
        REQUIRE(E == 0 || is_fp8(kI_dt) == (kI_scale != nullptr),
                "%s: kI_scale is required iff kI is E4M3", name);
    }
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1 && S <= csa::kMaxVarlenSeqs && kI_dt != CSA_DT_F32) {
            csa::VarlenMap map;
            map.S = S;
            int max_len = 0, max_n = 0;
            for (int s = 0; s <= S; ++s) {
                map.tok[s] = cu_seqlens[s];
                map.ent[s] = s == 0 ? 0 : map.ent[s - 1] + (cu_seqlens[s] - cu_seqlens[s - 1]) / m;
                if (s > 0) {
                    max_len = std::max(max_len, cu_seqlens[s] - cu_seqlens[s - 1]);
                    max_n = std::max(max_n, (cu_seqlens[s] - cu_seqlens[s - 1]) / m);
                }
            }
            if (max_len == 0) return ok();
            csa::IndexerArgs a{qI, qI_dt, qI_scale, kI, kI_dt, kI_scale, 1, max_len, H_I, d_I,
                               map.ent[S], nullptr, nullptr, m, topk, idx_out, hadamard_norm(d_I),
                               qI_weight};
            a.vl = &map;
            const cudaError_t ce = LAUNCH(csa::launch_indexer_packed(a, max_n, static_cast<cudaStream_t>(stream)));
            if (ce != cudaErrorNotSupported) return from_cuda(ce, name, nullptr);
            // otherwise: one launch per sequence below
        }
        long e = 0;
        for (int s = 0; s < S; ++s) {
            const int t0 = cu_seqlens[s], L = cu_seqlens[s + 1] - t0, N = L / m;
            const void* q = PTR_AT(qI, (long)t0 * H_I * d_I, dt_bytes(qI_dt));
            const float* qs = qI_scale ? qI_scale + (long)t0 * H_I : nullptr;
            const float* qw = qI_weight ? qI_weight + (long)t0 * H_I : nullptr;
            const void* k = PTR_AT(kI, e * d_I, dt_bytes(kI_dt));
            const float* ks = kI_scale ? kI_scale + e : nullptr;
            int* idx = idx_out ? idx_out + (long)t0 * topk : nullptr;
            if (pass == 0 && L > 0) {
                if (!(aligned16(q) && aligned16(k) && aligned4(idx) && (!qs || aligned4(qs)) &&
                      (!qw || aligned4(qw)) && (!ks || aligned4(ks))))
                    return fail(CSA_ERR_MISALIGNED, "%s: sequence %d's rows are not 16-byte aligned "
                                "(token offset %d, entry offset %ld)", name, s, t0, e);
            }
            if (pass == 1 && L > 0) {
                st = csa_indexer_topk(q, qI_dt, qs, qw, k, kI_dt, ks, 1, L, H_I, d_I, N, nullptr,
                                      nullptr, m, topk, idx, stream);
                if (st != CSA_OK) return st;
            }
            e += N;
        }
    }
    return ok();
}

static csa_status_t attn_varlen(const char* name, bool dense, const void* q, int dt, int S,
                                const int* cu, int H, int D, const void* kv_c, int m,
                                const int* idx, int topk, const void* kv_raw, int window,
                                float softmax_scale, void* out, float* lse_out, void* stream) {
    csa_status_t st = check_cu(name, S, cu, m);
    if (st != CSA_OK) return st;
    REQUIRE(is_dt(dt), "%s: unknown dtype", name);
    st = dense ? hca_dense_attn(q, dt, 0, 0, H, D, kv_c, 0, nullptr, m, kv_raw, 0, nullptr, nullptr,
                                window, nullptr, softmax_scale, out, lse_out, stream)
               : csa_sparse_attn(q, dt, 0, 0, H, D, kv_c, 0, idx, topk, kv_raw, 0, nullptr, nullptr,
                                 window, nullptr, softmax_scale, out, lse_out, stream);
    if (st != CSA_OK) return st;
    long E = 0;
    for (int s = 0; s < S; ++s) E += (cu[s + 1] - cu[s]) / m;
    REQUIRE(S == 0 || cu[S] == 0 || (q && out && kv_raw && (kv_c || E == 0) && (idx || topk == 0)),
            "%s: null tensor pointer", name);
    for (int pass = 0; pass < 2; ++pass) {
        if (pass == 1 && S <= csa::kMaxVarlenSeqs) {   // one launch, offsets by value
            csa::VarlenMap map;
            map.S = S;
            for (int s = 0; s <= S; ++s) {
                map.tok[s] = cu[s];
                map.ent[s] = s == 0 ? 0 : map.ent[s - 1] + (cu[s] - cu[s - 1]) / m;
            }
            const int T = cu[S];
            if (T == 0) return ok();
            csa::AttnArgs a{q, dt, 1, T, H, D, kv_c, map.ent[S], idx, dense ? 0 : topk,
                            nullptr, m, dense ? 1 : 0, kv_raw, T, nullptr, nullptr, window, nullptr,
                            softmax_scale > 0.0f ? softmax_scale : 1.0f / sqrtf((float)D), out,
                            lse_out};
            a.vl = &map;
            const cudaError_t ce = LAUNCH(csa::launch_attention_packed(a, static_cast<cudaStream_t>(stream)));
            if (ce != cudaErrorNotSupported) return from_cuda(ce, name, nullptr);
            // otherwise: one launch per sequence below
        }
        long e = 0;
        for (int s = 0; s < S; ++s) {
            const int t0 = cu[s], L = cu[s + 1] - t0, N = L / m;
            const size_t eb = dt_bytes(dt);
            const void* qs = PTR_AT(q, (long)t0 * H * D, eb);
            const void* kc = PTR_AT(kv_c, e * D, eb);
            const void* kr = PTR_AT(kv_raw, (long)t0 * D, eb);
            const int* ix = idx ? idx + (long)t0 * topk : nullptr;
            void* os = MPTR_AT(out, (long)t0 * H * D, eb);
            float* ls = lse_out ? lse_out + (long)t0 * H : nullptr;
            if (pass == 0 && L > 0) {
                if (!(aligned16(qs) && aligned16(kc) && aligned16(kr) && aligned16(os) &&
                      (!ix || aligned4(ix)) && (!ls || aligned4(ls))))
                    return fail(CSA_ERR_MISALIGNED, "%s: sequence %d's rows are not 16-byte aligned "
                                "(token offset %d, entry offset %ld)", name, s, t0, e);
            }
            if (pass == 1 && L > 0) {
                st = dense ? hca_dense_attn(qs, dt, 1, L, H, D, kc, N, nullptr, m, kr, L, nullptr,
                                            nullptr, window, nullptr, softmax_scale, os, ls, stream)
                           : csa_sparse_attn(qs, dt, 1, L, H, D, kc, N, ix, topk, kr, L, nullptr,
                                             nullptr, window, nullptr, softmax_scale, os, ls,
                                             stream);
                if (st != CSA_OK) return st;
            }
            e += N;
        }
    }
    return ok();
}

csa_status_t csa_sparse_attn_varlen(const void* q, int dt, int S, const int* cu_seqlens, int H,
                                    int D, const void* kv_c, int m, const int* idx, int topk,
                                    const void* kv_raw, int window, float softmax_scale, void* out,
                                    float* lse_out, void* stream) {
    return attn_varlen("csa_sparse_attn_varlen", false, q, dt, S, cu_seqlens, H, D, kv_c, m, idx,
                       topk, kv_raw, window, softmax_scale, out, lse_out, stream);
}

csa_status_t hca_dense_attn_varlen(const void* q, int dt, int S, const int* cu_seqlens, int H,
                                   int D, const void* kv_c, int m, const void* kv_raw, int window,
                                   float softmax_scale, void* out, float* lse_out, void* stream) {
    return attn_varlen("hca_dense_attn_varlen", true, q, dt, S, cu_seqlens, H, D, kv_c, m, nullptr,
                       0, kv_raw, window, softmax_scale, out, lse_out, stream);
}

}  // extern "C"
