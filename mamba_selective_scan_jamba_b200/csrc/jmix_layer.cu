// jm_layer_fwd: the full Mamba layer around the mixer core,
//   [x | z] = hidden . in_proj_w^T,  y = mixer(x, z),  out = y . out_proj_w^T
// (TransformerLens "Jamba" adapter page, "Architecture overview": in_proj /
// conv1d / x_proj / dt_proj / out_proj).  The two projections are plain dense
// GEMMs and go to cuBLASLt (bf16 in, fp32 accumulate, bf16 out), with the
// caller's workspace as its scratch: x and z are written as two separate
// [T, d_inner] matrices, the layout the mixer reads, and y feeds out_proj.
#include <cublasLt.h>
#include <string.h>

#include "jmix_internal.cuh"

#define JM_API extern "C" __attribute__((visibility("default")))

namespace jmix {
namespace {

constexpr size_t kLtWorkspace = size_t(32) << 20;

struct LayerWs {
  char* x;
  char* z;
  char* y;
  char* lt;
  char* mixer;
  size_t mixer_bytes;
  size_t bytes;
};

LayerWs layer_layout(int64_t T, int64_t d, size_t mixer_bytes, char* base) {
  LayerWs w{};
  size_t off = 0;
  auto take = [&](size_t n) {
    size_t o = off;
    off = align256(off + n);
    return base ? base + o : nullptr;
  };
  const size_t act = (size_t)T * (size_t)d * 2;
  // the mixer's workspace comes first: its error header is the layer's
  w.mixer = take(mixer_bytes);
  w.mixer_bytes = mixer_bytes;
  w.x = take(act);
  w.z = take(act);
  w.y = take(act);
  w.lt = take(kLtWorkspace);
  w.bytes = off;
  return w;
}

cublasLtHandle_t lt_handle() {
  static thread_local cublasLtHandle_t h = nullptr;
  if (!h && cublasLtCreate(&h) != CUBLAS_STATUS_SUCCESS) h = nullptr;
  return h;
}

// Out [M, N] = X [M, K] . W[N, K]^T, all row-major bf16, fp32 accumulation.
// In cuBLAS's column-major terms: Out^T [N, M] = op_T(W as K x N) . X^T (K x M).
jm_status lt_gemm(int64_t M, int64_t N, int64_t K, const void* X, const void* W, void* Out,
                  void* ws, size_t ws_bytes, cudaStream_t s) {
  cublasLtHandle_t h = lt_handle();
  if (!h) {
    set_error("cublasLtCreate failed");
    return JM_ERR_CUDA;
  }
  cublasLtMatmulDesc_t op = nullptr;
  cublasLtMatrixLayout_t la = nullptr, lb = nullptr, lc = nullptr;
  cublasLtMatmulPreference_t pref = nullptr;
  jm_status st = JM_ERR_CUDA;
  const cublasOperation_t ta = CUBLAS_OP_T, tb = CUBLAS_OP_N;
  const float alpha = 1.0f, beta = 0.0f;
  cublasLtMatmulHeuristicResult_t heur;
  int found = 0;
  if (cublasLtMatmulDescCreate(&op, CUBLAS_COMPUTE_32F, CUDA_R_32F) != CUBLAS_STATUS_SUCCESS ||
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta)) ||
      cublasLtMatmulDescSetAttribute(op, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb)) ||
      cublasLtMatrixLayoutCreate(&la, CUDA_R_16BF, (uint64_t)K, (uint64_t)N, K) ||
      cublasLtMatrixLayoutCreate(&lb, CUDA_R_16BF, (uint64_t)K, (uint64_t)M, K) ||
      cublasLtMatrixLayoutCreate(&lc, CUDA_R_16BF, (uint64_t)N, (uint64_t)M, N) ||
      cublasLtMatmulPreferenceCreate(&pref) ||
      cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES,
                                           &ws_bytes, sizeof(ws_bytes)) ||
      cublasLtMatmulAlgoGetHeuristic(h, op, la, lb, lc, lc, pref, 1, &heur, &found) ||
      found < 1) {
    set_error("cuBLASLt has no bf16 GEMM for %lld x %lld x %lld", (long long)M, (long long)N,
              (long long)K);
  } else if (cublasLtMatmul(h, op, &alpha, W, la, X, lb, &beta, Out, lc, Out, lc, &heur.algo, ws,
                            ws_bytes, s) != CUBLAS_STATUS_SUCCESS) {
    set_error("cublasLtMatmul failed (%lld x %lld x %lld)", (long long)M, (long long)N,
              (long long)K);
  } else {
    st = JM_OK;
  }
  if (pref) cublasLtMatmulPreferenceDestroy(pref);
  if (lc) cublasLtMatrixLayoutDestroy(lc);
  if (lb) cublasLtMatrixLayoutDestroy(lb);
  if (la) cublasLtMatrixLayoutDestroy(la);
  if (op) cublasLtMatmulDescDestroy(op);
  return st;
}

jm_status check_layer(const jm_dims* dims, int64_t d_model) {
  if (!dims) {
    set_error("dims is NULL");
    return JM_ERR_INVALID_ARG;
  }
  if (dims->io != JM_BF16) {
    set_error("jm_layer_fwd is built for bf16 io only");
    return JM_ERR_UNSUPPORTED;
  }
  if (d_model <= 0 || d_model % 8) {
    set_error("d_model must be a positive multiple of 8 (got %lld)", (long long)d_model);
    return JM_ERR_INVALID_ARG;
  }
  return JM_OK;
}

}  // namespace
}  // namespace jmix

using namespace jmix;

JM_API size_t jm_layer_fwd_workspace_size(const jm_dims* dims, int64_t d_model) {
  if (check_layer(dims, d_model) != JM_OK) return 0;
  const size_t mixer = jm_mixer_fwd_workspace_size(dims);
  if (!mixer) return 0;
  return layer_layout(dims->batch * dims->seqlen, dims->d_inner, mixer, nullptr).bytes;
}

JM_API jm_status jm_layer_fwd(const jm_dims* dims, int64_t d_model, const void* hidden,
                              const void* in_proj_w, const void* conv_w, const void* conv_b,
                              const void* xproj_w, const void* dt_norm_w, const void* b_norm_w,
                              const void* c_norm_w, const void* dtproj_w, const float* dt_bias,
                              const float* A_log, const float* D, const void* out_proj_w,
                              void* out, float* final_state, const void* init_conv_state,
                              const float* init_ssm_state, void* final_conv_state,
                              void* workspace, size_t ws_bytes, jm_stream_t stream) {
  jm_status st = check_layer(dims, d_model);
  if (st != JM_OK) return st;
  const size_t need = jm_layer_fwd_workspace_size(dims, d_model);
  if (!need)  // invalid mixer dims: the mixer's own check reports why (it launches nothing)
    return jm_mixer_fwd(dims, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                        nullptr, nullptr, nullptr, 0, stream);
  const int64_t T = dims->batch * dims->seqlen, d = dims->d_inner;
  const void* const ptrs[] = {hidden, in_proj_w, out_proj_w, out};
  const char* const names[] = {"hidden", "in_proj_w", "out_proj_w", "out"};
  for (int i = 0; i < 4; ++i) {
    if (T > 0 || i == 1 || i == 2) {
      if (!ptrs[i]) {
        set_error("%s is NULL", names[i]);
        return JM_ERR_INVALID_ARG;
      }
      if (reinterpret_cast<uintptr_t>(ptrs[i]) % 16) {
        set_error("%s is not 16-byte aligned", names[i]);
        return JM_ERR_INVALID_ARG;
      }
    }
  }
  if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || ws_bytes < need) {
    set_error("workspace must be 256-byte aligned and at least %zu bytes", need);
    return JM_ERR_WORKSPACE;
  }
  LayerWs w = layer_layout(T, d, jm_mixer_fwd_workspace_size(dims), static_cast<char*>(workspace));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const char* wi = static_cast<const char*>(in_proj_w);
  if (T > 0) {
    if ((st = lt_gemm(T, d, d_model, hidden, wi, w.x, w.lt, kLtWorkspace, s)) != JM_OK) return st;
    if ((st = lt_gemm(T, d, d_model, hidden, wi + (size_t)d * d_model * 2, w.z, w.lt, kLtWorkspace,
                      s)) != JM_OK)
      return st;
  }
  st = jm_mixer_fwd(dims, w.x, w.z, conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w,
                    dtproj_w, dt_bias, A_log, D, w.y, final_state, init_conv_state, init_ssm_state,
                    final_conv_state, w.mixer, w.mixer_bytes, stream);
  if (st != JM_OK) return st;
  if (T > 0 && (st = lt_gemm(T, d_model, d, w.y, out_proj_w, out, w.lt, kLtWorkspace, s)) != JM_OK)
    return st;
  return JM_OK;
}
