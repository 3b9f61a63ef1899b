// jm_layer_fwd: the full Mamba layer around the mixer core,
//   [x | z] = hidden . in_proj_w^T,  y = mixer(x, z),  out = y . out_proj_w^T
// (TransformerLens "Jamba" adapter page, "Architecture overview": in_proj /
// conv1d / x_proj / dt_proj / out_proj).  The two projections run on the
// tcgen05 GEMM of k_gemm.cu (bf16 in, fp32 accumulation, bf16 out): in_proj is
// one GEMM over N = 2 d_inner whose epilogue writes x and z as the two
// [T, d_inner] matrices the mixer reads; out_proj reads y.
#include <string.h>

#include "jmix_internal.cuh"

#define JM_API extern "C" __attribute__((visibility("default")))

namespace jmix {
namespace {

// Layer workspace: [error header][mixer workspace][x][z][y].  The projections
// record into the layer's header; out_proj carries the mixer's flags into it,
// so jm_poll_error on the layer workspace reports all three.
struct LayerWs {
  ErrFlags* hdr;
  char* x;
  char* z;
  char* y;
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
  w.hdr = reinterpret_cast<ErrFlags*>(take(sizeof(ErrFlags)));
  w.mixer = take(mixer_bytes);
  w.mixer_bytes = mixer_bytes;
  w.x = take(act);
  w.z = take(act);
  w.y = take(act);
  w.bytes = off;
  return w;
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
  cudaError_t e = cudaMemsetAsync(w.hdr, 0, sizeof(ErrFlags), s);
  if (e == cudaSuccess && T > 0)  // in_proj: N = 2 d_inner, x = columns [0, d), z = [d, 2d)
    e = gemm_bf16_tn(T, 2 * d, d_model, hidden, in_proj_w, w.x, w.z, d, w.hdr, nullptr, s, false);
  if (e != cudaSuccess) {
    set_error("in_proj: CUDA error: %s", cudaGetErrorString(e));
    return JM_ERR_CUDA;
  }
  st = jm_mixer_fwd(dims, w.x, w.z, conv_w, conv_b, xproj_w, dt_norm_w, b_norm_w, c_norm_w,
                    dtproj_w, dt_bias, A_log, D, w.y, final_state, init_conv_state, init_ssm_state,
                    final_conv_state, w.mixer, w.mixer_bytes, stream);
  if (st != JM_OK) return st;
  if (T > 0) {  // (with no tokens nothing ran that could set a flag)
    e = gemm_bf16_tn(T, d_model, d, w.y, out_proj_w, out, nullptr, d_model, w.hdr,
                     reinterpret_cast<const ErrFlags*>(w.mixer), s, true);
    if (e != cudaSuccess) {
      set_error("out_proj: CUDA error: %s", cudaGetErrorString(e));
      return JM_ERR_CUDA;
    }
  }
  return JM_OK;
}
