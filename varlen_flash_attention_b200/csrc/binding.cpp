// Compiled argument marshalling for the hottest entry point,
// attn_fwd_split_kv: shape, dtype, device and layout checks on the torch
// tensors, sk_tensor_t descriptors, the current stream, then the C ABI call.
// No computation happens here (every step of the attention runs in the
// library's kernels); the point is the host cost of a call, which through
// Python-level attribute access and ctypes is several times the C ABI's own.
// Errors are raised as ValueError / TypeError with the same wording as the
// Python checks; a non-OK status from the library is returned to the caller,
// which raises SplitKVError.
#include <c10/cuda/CUDAGuard.h>
#include <c10/cuda/CUDAStream.h>
#include <dlfcn.h>
#include <torch/extension.h>

#include <optional>
#include <string>
#include <vector>

#include "../../include/splitkv_attn.h"

namespace {

// The library's entry points, resolved from the file the Python binding
// loaded (dlopen of the same path returns the same instance).
using split_fn = decltype(&attn_fwd_split_kv);
using split_ex_fn = decltype(&attn_fwd_split_kv_ex);
split_fn g_split = nullptr;
split_ex_fn g_split_ex = nullptr;

void bind_library(const std::string& path) {
  void* h = dlopen(path.c_str(), RTLD_NOW | RTLD_GLOBAL);
  if (!h) throw std::runtime_error(std::string("cannot load ") + path + ": " + dlerror());
  g_split = reinterpret_cast<split_fn>(dlsym(h, "attn_fwd_split_kv"));
  g_split_ex = reinterpret_cast<split_ex_fn>(dlsym(h, "attn_fwd_split_kv_ex"));
  if (!g_split || !g_split_ex) throw std::runtime_error("attn_fwd_split_kv entry points missing in " + path);
}

sk_tensor_t desc_of(const at::Tensor& t) {
  sk_tensor_t d;
  d.ptr = t.numel() > 0 ? t.data_ptr() : nullptr;
  d.stride_b = t.stride(0);
  d.stride_s = t.stride(1);
  d.stride_h = t.stride(2);
  d.len_s = static_cast<int32_t>(t.size(1));
  return d;
}

std::string shape_str(const at::Tensor& t) {
  std::string s = "(";
  for (int64_t i = 0; i < t.dim(); ++i) s += (i ? ", " : "") + std::to_string(t.size(i));
  return s + (t.dim() == 1 ? ",)" : ")");
}

void check4(const at::Tensor& t, const char* name, const at::Device& dev) {
  if (t.dim() != 4) throw pybind11::value_error(std::string(name) + " must be [batch, seq, heads, head_dim]");
  if (t.scalar_type() != at::kBFloat16) throw pybind11::type_error("expected bf16");
  if (t.size(3) > 1 && t.stride(3) != 1) throw pybind11::value_error("head_dim must be contiguous (stride 1)");
  if (t.numel() > 0) {
    if (!t.is_cuda()) throw pybind11::value_error("expected a CUDA tensor");
    if (t.device() != dev)
      throw pybind11::value_error(std::string(name) + " is on " + t.device().str() + ", expected " + dev.str() +
                                  " (the device of q)");
  }
}

// Returns the library's status (0 = OK).
int attn_fwd_split_kv_call(const at::Tensor& q, const at::Tensor& kp, const at::Tensor& vp, const at::Tensor& ks,
                           const at::Tensor& vs, const at::Tensor& out,
                           const std::optional<std::vector<int32_t>>& real_len,
                           const std::optional<std::vector<int32_t>>& q_valid, double scale, int64_t stream) {
  if (!g_split) throw std::runtime_error("library not bound (bind_library)");
  if (q.dim() != 4) throw pybind11::value_error("q must be [batch, seq, heads, head_dim]");
  const int64_t B = q.size(0), Hq = q.size(2), D = q.size(3);
  const at::Tensor* kv[4] = {&kp, &vp, &ks, &vs};
  const char* names[4] = {"k_prefix", "v_prefix", "k_suffix", "v_suffix"};
  int64_t Hkv = -1;
  for (int i = 0; i < 4; ++i) {
    const at::Tensor& t = *kv[i];
    if (t.dim() != 4) throw pybind11::value_error(std::string(names[i]) + " must be [batch, seq, kv_heads, head_dim]");
    if (t.size(0) != B || t.size(3) != D)
      throw pybind11::value_error(std::string(names[i]) + " " + shape_str(t) + ": batch and head_dim must match q " +
                                  shape_str(q));
    if (Hkv < 0) Hkv = t.size(2);
    else if (t.size(2) != Hkv)
      throw pybind11::value_error(std::string(names[i]) + " has " + std::to_string(t.size(2)) +
                                  " heads, the other K/V tensors " + std::to_string(Hkv));
  }
  if (kp.size(1) != vp.size(1) || ks.size(1) != vs.size(1))
    throw pybind11::value_error("k and v of the prefix (and of the suffix) must have the same length");
  if (!out.sizes().equals(q.sizes()))
    throw pybind11::value_error("out " + shape_str(out) + " must have q's shape " + shape_str(q));
  const at::Device dev = q.device();
  check4(q, "q", dev);
  for (int i = 0; i < 4; ++i) check4(*kv[i], names[i], dev);
  check4(out, "out", dev);
  if (real_len && static_cast<int64_t>(real_len->size()) != B)
    throw pybind11::value_error("expected " + std::to_string(B) + " values, got " + std::to_string(real_len->size()));
  if (q_valid && static_cast<int64_t>(q_valid->size()) != B)
    throw pybind11::value_error("expected " + std::to_string(B) + " values, got " + std::to_string(q_valid->size()));
  sk_tensor_t d[6] = {desc_of(q), desc_of(kp), desc_of(vp), desc_of(ks), desc_of(vs), desc_of(out)};
  const int32_t* rl = real_len ? real_len->data() : nullptr;
  // The library launches on the current device; switch only when q lives elsewhere.
  std::optional<c10::cuda::CUDAGuard> guard;
  if (dev.is_cuda() && dev.index() != c10::cuda::current_device()) guard.emplace(dev.index());
  void* s = stream != 0 ? reinterpret_cast<void*>(stream)
                        : (dev.is_cuda() ? static_cast<void*>(c10::cuda::getCurrentCUDAStream(dev.index()).stream())
                                         : nullptr);
  const int32_t b32 = static_cast<int32_t>(B), hq = static_cast<int32_t>(Hq), hkv = static_cast<int32_t>(Hkv);
  const int32_t d32 = static_cast<int32_t>(D);
  if (q_valid)
    return g_split_ex(&d[0], &d[1], &d[2], &d[3], &d[4], rl, hq, hkv, static_cast<float>(scale), &d[5], b32, d32,
                      q_valid->data(), s);
  return g_split(&d[0], &d[1], &d[2], &d[3], &d[4], rl, hq, hkv, static_cast<float>(scale), &d[5], b32, d32, s);
}

}  // namespace

PYBIND11_MODULE(TORCH_EXTENSION_NAME, m) {
  m.def("bind_library", &bind_library, "resolve the C ABI entry points from the library file", pybind11::arg("path"));
  m.def("attn_fwd_split_kv", &attn_fwd_split_kv_call, "attn_fwd_split_kv through the C ABI (argument marshalling only)",
        pybind11::arg("q"), pybind11::arg("k_prefix"), pybind11::arg("v_prefix"), pybind11::arg("k_suffix"),
        pybind11::arg("v_suffix"), pybind11::arg("out"), pybind11::arg("real_len"), pybind11::arg("q_valid"),
        pybind11::arg("softmax_scale"), pybind11::arg("stream"));
}
