// layer.cu -- one Gated DeltaNet layer forward under NVFP4 W4A4, composed on
// one stream from the library's kernels (review page of "Why Gated DeltaNet
// Survives 4-Bit Quantization": NVFP4 W4A4 on every linear module of the GDN
// block, paper sec.3; fused in_proj with one harmonised weight scale, sec.6):
//
//   x (bf16) -> NVFP4 -> fused in_proj GEMM -> P = q|k|v|z|a|b (f32)
//   P -> gates (g, beta) and L2-normalised q, k
//   -> delta-rule scan (state in / out) -> o (f32)
//   o -> NVFP4 -> out_proj GEMM -> y (f32)
//
// No host synchronisation inside: the per-tensor scales stay on the device.
#include "common.cuh"

namespace nvg {

nvfp4_status validate_tensor(const nvfp4_tensor* t, const char* name);
nvfp4_status validate_dims(const gdn_dims* d);
nvfp4_status zero_words_launch(unsigned int* w, int n, cudaStream_t st);
nvfp4_status short_conv_launch(const float* x, int64_t ld_x, int B, int64_t T, int C, int W, const float* w,
                               const float* state_in, float* state_out, float* out, int64_t ld_out, cudaStream_t st);
nvfp4_status l2norm_launch(const float* proj, int64_t ld, int64_t n, const gdn_dims& d, float* q_hat, float* k_hat,
                           cudaStream_t st);
nvfp4_status output_gate_launch(const float* o, const float* z, int64_t ld_z, const float* w, int64_t n, int Hv, int V,
                                float* out, unsigned int* amax_word, cudaStream_t st);
nvfp4_status quantize_launch(const void* x, int32_t x_dtype, int64_t rows, int64_t cols, int64_t ld,
                             const nvfp4_tensor& out, int32_t flags, void* workspace, cudaStream_t st);
nvfp4_status gemm_launch(const nvfp4_tensor& A, const nvfp4_tensor& B, float* C, int64_t ldc, cudaStream_t st);
nvfp4_status gate_only_launch(const float* proj, int64_t ld, int64_t n, const gdn_dims& d, const float* A_log,
                              const float* dt_bias, float* g, float* beta, cudaStream_t st);
nvfp4_status gates_launch(const float* proj, int64_t ld, int64_t n, const gdn_dims& d, const float* A_log,
                          const float* dt_bias, float* q_hat, float* k_hat, float* g, float* beta, cudaStream_t st);
size_t scan_workspace_bytes(int B, int64_t T, const gdn_dims& d, int algo);
nvfp4_status scan_launch(const float* q, const float* k, const float* v, int64_t ld_v, const float* g,
                         const float* beta, int B, int64_t T, const gdn_dims& d, float scale, int form, int algo,
                         const float* s_in, float* s_out, float* o, void* ws, cudaStream_t st,
                         unsigned int* o_amax, int64_t ld_qk, int normalize_qk);

static int64_t n_in_of(const gdn_dims& d) { return 2ll * d.Hk * d.K + 2ll * d.Hv * d.V + 2ll * d.Hv; }
static int64_t ld_proj_of(const gdn_dims& d) { return (n_in_of(d) + 3) / 4 * 4; }
static int64_t qkv_width(const gdn_dims& d) { return 2ll * d.Hk * d.K + static_cast<int64_t>(d.Hv) * d.V; }

static nvfp4_status layout_of(const gdn_layer_weights* w, int32_t B, int64_t T, gdn_layer_ws_layout* L) {
    const gdn_dims& d = w->dims;
    const int64_t BT = static_cast<int64_t>(B) * T, H = w->hidden, HvV = static_cast<int64_t>(d.Hv) * d.V;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~size_t(255);
        return at;
    };
    L->x_codes = take(BT * H / 2);
    L->x_sf = take(nvfp4_sf_bytes(BT, H));
    L->x_scale = take(4);
    L->proj = take(BT * ld_proj_of(d) * 4);
    L->q_hat = take(BT * d.Hk * d.K * 4);
    L->k_hat = take(BT * d.Hk * d.K * 4);
    L->g = take(BT * d.Hv * 4);
    L->beta = take(BT * d.Hv * 4);
    L->o = take(BT * HvV * 4);
    L->o_gated = take(w->out_norm ? BT * HvV * 4 : 0);
    L->qkv_conv = take(w->conv_weight ? BT * qkv_width(d) * 4 : 0);
    L->o_codes = take(BT * HvV / 2);
    L->o_sf = take(nvfp4_sf_bytes(BT, HvV));
    L->o_scale = take(4);
    L->quant_ws = take(nvfp4_quantize_workspace_size());
    L->scan_ws = take(scan_workspace_bytes(B, T, d, GDN_SCAN_AUTO));
    L->total = off;
    return NVFP4_OK;
}

static nvfp4_status validate_layer(const gdn_layer_weights* w, int32_t B, int64_t T) {
    if (!w) return fail(NVFP4_ERR_INVALID_ARG, "weights is null");
    nvfp4_status s = validate_dims(&w->dims);
    if (s != NVFP4_OK) return s;
    if ((s = validate_tensor(&w->w_in, "w_in")) != NVFP4_OK) return s;
    if ((s = validate_tensor(&w->w_out, "w_out")) != NVFP4_OK) return s;
    if (!w->A_log || !w->dt_bias) return fail(NVFP4_ERR_INVALID_ARG, "A_log / dt_bias null");
    if (w->out_norm && !aligned16(w->out_norm)) return fail(NVFP4_ERR_MISALIGNED, "out_norm must be 16-byte aligned");
    if (w->conv_weight && (w->conv_width < 2 || w->conv_width > 4))
        return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "conv_width must be 2, 3 or 4");
    if (w->hidden < 64 || w->hidden % 64) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "hidden must be a multiple of 64");
    if (w->w_in.rows != n_in_of(w->dims) || w->w_in.cols != w->hidden)
        return fail(NVFP4_ERR_INVALID_ARG, "w_in must be [2HkK + 2HvV + 2Hv, hidden]");
    if (w->w_out.rows != w->hidden || w->w_out.cols != static_cast<int64_t>(w->dims.Hv) * w->dims.V)
        return fail(NVFP4_ERR_INVALID_ARG, "w_out must be [hidden, Hv*V]");
    if (B < 1 || T < 1) return fail(NVFP4_ERR_INVALID_ARG, "B and T must be >= 1");
    if (static_cast<int64_t>(B) * T > (int64_t(1) << 30)) return fail(NVFP4_ERR_UNSUPPORTED_SHAPE, "B*T too large");
    return NVFP4_OK;
}

}  // namespace nvg

extern "C" nvfp4_status gdn_layer_workspace_layout(const gdn_layer_weights* w, int32_t B, int64_t T,
                                                   gdn_layer_ws_layout* out) {
    using namespace nvg;
    nvfp4_status s = validate_layer(w, B, T);
    if (s != NVFP4_OK) return s;
    if (!out) return fail(NVFP4_ERR_INVALID_ARG, "out is null");
    return layout_of(w, B, T, out);
}

extern "C" nvfp4_status gdn_layer_forward(const gdn_layer_weights* w, const void* x_bf16, int32_t B, int64_t T,
                                          float* y, const float* state_in, float* state_out, int32_t form,
                                          void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
    return gdn_layer_forward_stateful(w, x_bf16, B, T, y, state_in, state_out, nullptr, nullptr, form, workspace,
                                      workspace_bytes, stream);
}

namespace nvg {
// The layer's launches; with events (an array of kLayerEvents cudaEvent_t), event
// i is recorded before stage i (quantise x, in_proj, gates and the optional
// convolution, scan, the optional output gate and quantise o, out_proj) and the
// last one after out_proj.
constexpr int kLayerEvents = 7;
static nvfp4_status layer_forward(const gdn_layer_weights* w, const void* x_bf16, int32_t B, int64_t T, float* y,
                                  const float* state_in, float* state_out, const float* conv_state_in,
                                  float* conv_state_out, int32_t form, void* workspace, size_t workspace_bytes,
                                  nvfp4_stream_t stream, void* const* events) {
    nvfp4_status s = validate_layer(w, B, T);
    if (s != NVFP4_OK) return s;
    if (!x_bf16 || !y) return fail(NVFP4_ERR_INVALID_ARG, "x / y null");
    if (form != GDN_FORM_PAGES && form != GDN_FORM_STANDARD) return fail(NVFP4_ERR_INVALID_ARG, "bad form");
    if (!aligned16(x_bf16) || !aligned16(y)) return fail(NVFP4_ERR_MISALIGNED, "x / y must be 16-byte aligned");
    if (!aligned16(state_in) || !aligned16(state_out))
        return fail(NVFP4_ERR_MISALIGNED, "state_in and state_out must be 16-byte aligned");
    gdn_layer_ws_layout L;
    layout_of(w, B, T, &L);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
        return fail(NVFP4_ERR_WORKSPACE, "layer workspace missing, too small or not 256-byte aligned");
    cudaStream_t st = as_stream(stream);
    auto mark = [&](int i) -> nvfp4_status {
        if (!events) return NVFP4_OK;
        const cudaError_t e = cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st);
        return e == cudaSuccess ? NVFP4_OK : cuda_fail(e, "stage event record");
    };
    char* ws = static_cast<char*>(workspace);
    const gdn_dims& d = w->dims;
    const int64_t BT = static_cast<int64_t>(B) * T, H = w->hidden, HvV = static_cast<int64_t>(d.Hv) * d.V;
    const int64_t ldp = ld_proj_of(d);

    nvfp4_tensor xq{reinterpret_cast<uint8_t*>(ws + L.x_codes), reinterpret_cast<uint8_t*>(ws + L.x_sf),
                    reinterpret_cast<float*>(ws + L.x_scale), BT, H};
    nvfp4_tensor oq{reinterpret_cast<uint8_t*>(ws + L.o_codes), reinterpret_cast<uint8_t*>(ws + L.o_sf),
                    reinterpret_cast<float*>(ws + L.o_scale), BT, HvV};
    float* proj = reinterpret_cast<float*>(ws + L.proj);
    float* g = reinterpret_cast<float*>(ws + L.g);
    float* beta = reinterpret_cast<float*>(ws + L.beta);
    float* o = reinterpret_cast<float*>(ws + L.o);

    // quantiser words: [0] x amax, [1] x arrival counter, [2] o amax, [3] gated-o amax,
    // zeroed by one small kernel (it chains with its neighbours by programmatic launch)
    unsigned int* qw = reinterpret_cast<unsigned int*>(ws + L.quant_ws);
    if ((s = mark(0)) != NVFP4_OK) return s;
    if ((s = zero_words_launch(qw, 4, st)) != NVFP4_OK) return s;
    if ((s = quantize_launch(x_bf16, NVFP4_DTYPE_BF16, BT, H, H, xq, kQuantComputeZeroedWs, qw, st)) != NVFP4_OK)
        return s;
    if ((s = mark(1)) != NVFP4_OK) return s;
    if ((s = gemm_launch(xq, w->w_in, proj, ldp, st)) != NVFP4_OK) return s;
    if ((s = mark(2)) != NVFP4_OK) return s;
    // q|k|v come from the projection, or from its short convolution when one is set
    const float* qkv = proj;
    int64_t ld_qkv = ldp;
    if (w->conv_weight) {
        float* cv = reinterpret_cast<float*>(ws + L.qkv_conv);
        if ((s = short_conv_launch(proj, ldp, B, T, static_cast<int>(qkv_width(d)), w->conv_width, w->conv_weight,
                                   conv_state_in, conv_state_out, cv, qkv_width(d), st)) != NVFP4_OK)
            return s;
        qkv = cv;
        ld_qkv = qkv_width(d);
    }
    // Both scans read the raw q, k slices and normalise them themselves (the
    // chunked one while staging a chunk, the recurrent one per token), so only g
    // and beta are formed here.
    const bool chunked = T > 1;
    if ((s = gate_only_launch(proj, ldp, BT, d, w->A_log, w->dt_bias, g, beta, st)) != NVFP4_OK) return s;
    const float* q_in = qkv;
    const float* k_in = qkv + static_cast<int64_t>(d.Hk) * d.K;
    const int64_t ld_qk = ld_qkv;
    const float scale = 1.0f / sqrtf(static_cast<float>(d.K));
    // the scan folds max|o| into the quantiser's amax word as it writes o, so the o
    // quantiser runs its quantisation pass only
    unsigned int* o_amax = qw + 2;
    if ((s = mark(3)) != NVFP4_OK) return s;
    if ((s = scan_launch(q_in, k_in, qkv + 2ll * d.Hk * d.K, ld_qkv, g, beta, B, T, d, scale, form,
                         chunked ? GDN_SCAN_CHUNKED : GDN_SCAN_RECURRENT, state_in, state_out, o, ws + L.scan_ws, st,
                         o_amax, ld_qk, 1)) != NVFP4_OK)
        return s;
    if ((s = mark(4)) != NVFP4_OK) return s;
    const float* oq_in = o;
    unsigned int* oq_amax = o_amax;
    if (w->out_norm) {
        // output gate: G = RMSNorm(o) * w * SiLU(z), its amax into the fourth word
        float* og = reinterpret_cast<float*>(ws + L.o_gated);
        const float* z = proj + 2ll * d.Hk * d.K + static_cast<int64_t>(d.Hv) * d.V;
        if ((s = output_gate_launch(o, z, ldp, w->out_norm, BT, d.Hv, d.V, og, qw + 3, st)) != NVFP4_OK) return s;
        oq_in = og;
        oq_amax = qw + 3;
    }
    if ((s = quantize_launch(oq_in, NVFP4_DTYPE_FP32, BT, HvV, HvV, oq, kQuantFromAmax, oq_amax, st)) != NVFP4_OK)
        return s;
    if ((s = mark(5)) != NVFP4_OK) return s;
    if ((s = gemm_launch(oq, w->w_out, y, H, st)) != NVFP4_OK) return s;
    return mark(6);
}
}  // namespace nvg

extern "C" nvfp4_status gdn_layer_forward_stateful(const gdn_layer_weights* w, const void* x_bf16, int32_t B,
                                                   int64_t T, float* y, const float* state_in, float* state_out,
                                                   const float* conv_state_in, float* conv_state_out, int32_t form,
                                                   void* workspace, size_t workspace_bytes, nvfp4_stream_t stream) {
    return nvg::layer_forward(w, x_bf16, B, T, y, state_in, state_out, conv_state_in, conv_state_out, form,
                              workspace, workspace_bytes, stream, nullptr);
}

extern "C" nvfp4_status gdn_layer_forward_timed(const gdn_layer_weights* w, const void* x_bf16, int32_t B,
                                                int64_t T, float* y, const float* state_in, float* state_out,
                                                const float* conv_state_in, float* conv_state_out, int32_t form,
                                                void* workspace, size_t workspace_bytes, nvfp4_stream_t stream,
                                                void* const* events) {
    using namespace nvg;
    if (!events) return fail(NVFP4_ERR_INVALID_ARG, "events is null");
    for (int i = 0; i < kLayerEvents; ++i)
        if (!events[i]) return fail(NVFP4_ERR_INVALID_ARG, "event handle is null");
    return layer_forward(w, x_bf16, B, T, y, state_in, state_out, conv_state_in, conv_state_out, form, workspace,
                         workspace_bytes, stream, events);
}
