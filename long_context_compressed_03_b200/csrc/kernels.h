// kernels.h -- internal launch interface between the C ABI and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace csa {

// A paged cache.  Logical entry s (0 <= s < N_cap = max_pages * page size) of
// batch element b is physical row
//   bt[b * max_pages + (s >> page_shift)] * page size + (s & (page size - 1))
// of the page pool; bt == nullptr means the plain layout, row b * N_cap + s.
struct PageMap {
    const int* bt = nullptr;
    int max_pages = 0;
    int page_shift = 0;
    int num_pages = 0;         // pool size in pages: page ids outside [0, num_pages) are absent
};

// Physical row of logical entry s of element b, or -1 when its page id lies
// outside the pool (the entry is then treated as absent: never read or written).
__host__ __device__ __forceinline__ long cache_row(const PageMap& pm, int N_cap, int b, int s) {
    if (!pm.bt) return (long)b * N_cap + s;
    const int pg = pm.bt[(size_t)b * pm.max_pages + (s >> pm.page_shift)];
    if (pg < 0 || pg >= pm.num_pages) return -1;
    return ((long)pg << pm.page_shift) + (s & ((1 << pm.page_shift) - 1));
}

// Packed sequences handed to one launch: sequence s owns tokens
// [tok[s], tok[s+1]) and compressed entries [ent[s], ent[s+1]).  Passed by
// value in the kernel parameters (no device buffer); S == 0: not packed.
constexpr int kMaxVarlenSeqs = 128;
struct VarlenMap {
    int S = 0;
    int tok[kMaxVarlenSeqs + 1];
    int ent[kMaxVarlenSeqs + 1];
    int uoff[kMaxVarlenSeqs + 1];   // prefill attention: first 4-token unit of each sequence
};

struct CompressArgs {
    const void* x; int x_dt;
    int B, n, d_in;
    const void* W; int d_out;
    int m, overlap;
    void* out; int out_dt;
    float* out_row_scale;
    int N_c;
    float hnorm;               // fp32(1/sqrt(d_out)) for the Hadamard fp8 type
    const VarlenMap* vl = nullptr;   // packed: B = S, n = longest, N_c = most entries
};

struct GatedArgs {
    const void* x; int x_dt;
    int B, n, d_in;
    const void* W_kv;          // [d_in, c*d_out], x_dt
    const void* W_gate;        // [d_in, c*d_out], x_dt
    const float* ape;          // [m, c*d_out]
    int d_out, m, overlap;     // c = 2 if overlap else 1
    void* out; int out_dt;
    float* out_row_scale;
    int N_c;
    float hnorm;
};

struct AppendArgs {
    const void* x; int x_dt;
    int B, d_in;
    const void* W; int d_out;
    int m, overlap;
    const int* pos;
    float* state;
    void* cache; int out_dt;
    float* cache_scale;
    int N_cap;
    int* n_entries;
    float hnorm;               // fp32(1/sqrt(d_out)) for the Hadamard fp8 type
    PageMap pages;             // cache (and cache_scale) layout
};

struct IndexerArgs {
    const void* qI; int qI_dt; const float* qI_scale;
    const void* kI; int kI_dt; const float* kI_scale;
    int B, n_q, H_I, d_I, N_cap;
    const int* n_entries; const int* q_pos;
    int m, topk;
    int* idx_out;
    float hnorm;               // fp32(1/sqrt(d_I)): keys of the Hadamard fp8 type
    const float* qI_weight;    // [B, n_q, H_I] gate weights or NULL (all 1)
    PageMap pages;             // kI (and kI_scale) layout
    const VarlenMap* vl = nullptr;   // packed (tensor-core kernel only): B = S, n_q = longest,
                                     // N_cap = total entries
    int pos0 = 0;              // q_pos == NULL: query q of every element sits at pos0 + q
};

struct AttnArgs {
    const void* q; int dt;
    int B, n_q, H, D;
    const void* kv_c; int N_cap;
    const int* idx; int topk;         // sparse mode
    const int* n_entries; int m;      // dense (HCA) mode
    int dense;
    const void* kv_raw; int L_raw;
    const int* raw_pos0; const int* raw_len;
    int window;
    const int* q_pos;
    float scale;
    void* out; float* lse_out;
    PageMap pages;             // kv_c layout
    const VarlenMap* vl = nullptr;   // packed (tensor-core kernel only): B = 1, n_q = L_raw = T
                                     // tokens, N_cap = total entries
    int pos0 = 0;              // q_pos == NULL: query q of every element sits at pos0 + q
    int raw_base = 0;          // raw_pos0 == NULL: raw row j of every element holds position raw_base + j
};

// Device address of this library's error word on the current device (set by
// kernels whose bounded waits expired; read back by csa_check_device_error).
uint32_t* device_error_word();

// Time limit (ns) of each bounded wait of the tensor-core kernels' work,
// 1 s unless a test set a shorter one (csa_debug_set_wait_limit).
uint64_t wait_limit_ns();
void set_wait_limit_ns(uint64_t ns);
// One-shot test hook: the next tensor-core launch makes one thread of every
// CTA wait on a barrier that nothing completes, so that wait runs out.
int take_stall();
void set_stall(int on);

// tcgen05 prefill attention (64 heads x 128, bf16, positions 0..n-1).
bool attention_tc_supported(const AttnArgs& a);
cudaError_t launch_attention_tc(const AttnArgs& a, uint32_t* err, cudaStream_t s);

// tcgen05 attention for few query rows (decode): bf16, 64 heads x 128, the
// score tile transposed (128 keys x 64 heads), one row's key tiles dealt over
// a thread-block cluster sized so that every cluster is resident at once.
bool attention_dec_tc_supported(const AttnArgs& a);
cudaError_t launch_attention_dec_tc(const AttnArgs& a, uint32_t* err, cudaStream_t s);

// tcgen05 indexer + fused exact top-k for prefill (d_I = 64, H_I <= 4).
bool indexer_tc_supported(const IndexerArgs& a);
cudaError_t launch_indexer_tc(const IndexerArgs& a, uint32_t* err, cudaStream_t s);

// Cluster split-KV attention for few query rows (decode): bf16, D in {64, 128},
// H in {16, 32, 64, 128}.
bool attention_split_supported(const AttnArgs& a);
cudaError_t launch_attention_split(const AttnArgs& a, cudaStream_t s);

// Cluster split indexer + exact top-k for few query rows (decode): fp8 keys
// with per-row scales, d_I in {64, 128}, H_I <= 8.
bool indexer_split_supported(const IndexerArgs& a);
cudaError_t launch_indexer_split(const IndexerArgs& a, cudaStream_t s);

// Counts one kernel launch (read back through csa_kernel_launches()).
void count_launch();

// Each returns cudaSuccess or the launch error; `why` receives a static
// reason string when the configuration is unsupported (returned as
// cudaErrorNotSupported).
cudaError_t launch_compress(const CompressArgs& a, cudaStream_t s, const char** why);
// One launch over packed sequences (a.vl, a.B = 1, a.N_cap = total entries,
// a.n_q = longest sequence), or cudaErrorNotSupported when the tensor-core
// indexer does not serve the per-sequence shape (max_entries entries).
cudaError_t launch_indexer_packed(const IndexerArgs& a, int max_entries, cudaStream_t s);
// One launch over packed sequences (a.vl set), or cudaErrorNotSupported when
// the tensor-core attention does not serve the shape.
cudaError_t launch_attention_packed(const AttnArgs& a, cudaStream_t s);
cudaError_t launch_compress_gated(const GatedArgs& a, cudaStream_t s, const char** why);
cudaError_t launch_compress_append(const AppendArgs& a, cudaStream_t s, const char** why);
cudaError_t launch_indexer_topk(const IndexerArgs& a, cudaStream_t s, const char** why);
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s, const char** why);

}  // namespace csa
