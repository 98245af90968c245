// fp8gemm_jit.h -- runtime specialisation of the tiled kernel (host side).
//
// The pages' library compiles its kernels at run time with the GEMM shape as compile-time
// constants (the chattools.cn explainer and the flashmla.org product page, "JIT" design ideas).
// Here that is an opt-in second path next to the ahead-of-time build: on the first call of a
// shape, the kernel sources this library was built from (embedded at build time) are compiled
// with NVRTC for sm_100a with -DFG_JIT_* constants -- K blocks, K, N, sfb blocks, tile columns and
// the tile-walk grouping -- loaded as a module through the driver API, cached per device and
// shape, and launched exactly like the ahead-of-time kernel (same arguments, same programmatic
// dependent launch attribute).  NVRTC and the driver entry points are resolved at run time, so the
// library has no link-time dependency on either; without them the JIT path reports
// FG_ERR_UNSUPPORTED and nothing else changes.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <dlfcn.h>

#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

namespace fgjit {

// nvrtc entry points (resolved with dlopen; nvrtcResult is an int enum, programs are opaque)
typedef int (*CreateProgramFn)(void**, const char*, const char*, int, const char* const*, const char* const*);
typedef int (*AddNameFn)(void*, const char*);
typedef int (*CompileFn)(void*, int, const char* const*);
typedef int (*LoweredNameFn)(void*, const char*, const char**);
typedef int (*SizeFn)(void*, size_t*);
typedef int (*GetBytesFn)(void*, char*);
typedef int (*DestroyFn)(void**);

// driver entry points used for the runtime-compiled modules
typedef CUresult (*ModuleLoadDataFn)(CUmodule*, const void*);
typedef CUresult (*ModuleGetFunctionFn)(CUfunction*, CUmodule, const char*);
typedef CUresult (*FuncSetAttributeFn)(CUfunction, CUfunction_attribute, int);
typedef CUresult (*FuncGetAttributeFn)(int*, CUfunction_attribute, CUfunction);
typedef CUresult (*LaunchKernelExFn)(const CUlaunchConfig*, CUfunction, void**, void**);

struct Api {
  bool tried = false;
  bool ok = false;
  CreateProgramFn create = nullptr;
  AddNameFn add_name = nullptr;
  CompileFn compile = nullptr;
  LoweredNameFn lowered = nullptr;
  SizeFn cubin_size = nullptr;
  GetBytesFn cubin = nullptr;
  SizeFn log_size = nullptr;
  GetBytesFn log = nullptr;
  DestroyFn destroy = nullptr;
  ModuleLoadDataFn module_load = nullptr;
  ModuleGetFunctionFn get_function = nullptr;
  FuncSetAttributeFn set_attr = nullptr;
  FuncGetAttributeFn get_attr = nullptr;
  LaunchKernelExFn launch = nullptr;
  std::string include_dir;  // CUDA headers for NVRTC (cuda_bf16.h)
};

inline Api& api() {
  static Api a;
  return a;
}

template <typename F>
bool sym(void* h, const char* name, F* out) {
  *out = reinterpret_cast<F>(dlsym(h, name));
  return *out != nullptr;
}

template <typename F>
bool drv(const char* name, F* out) {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return false;
  *out = reinterpret_cast<F>(fn);
  return fn != nullptr;
}

// Resolve NVRTC and the CUDA headers once (caller holds a lock); the driver entry points are
// resolved separately (load_driver), so that compiling needs no GPU.
inline bool load_api() {
  Api& a = api();
  if (a.tried) return a.ok;
  a.tried = true;
  std::vector<std::string> roots;
  if (const char* h = std::getenv("CUDA_HOME")) roots.push_back(h);
  roots.push_back("/usr/local/cuda");
  void* h = nullptr;
  for (const std::string& r : roots) {
    const std::string inc = r + "/include/cuda_bf16.h";
    if (FILE* f = std::fopen(inc.c_str(), "r")) {
      std::fclose(f);
      if (a.include_dir.empty()) a.include_dir = r + "/include";
    }
    if (!h) h = dlopen((r + "/lib64/libnvrtc.so.12").c_str(), RTLD_NOW | RTLD_LOCAL);
  }
  if (!h) h = dlopen("libnvrtc.so.12", RTLD_NOW | RTLD_LOCAL);
  if (!h || a.include_dir.empty()) return false;
  a.ok = sym(h, "nvrtcCreateProgram", &a.create) && sym(h, "nvrtcAddNameExpression", &a.add_name) &&
         sym(h, "nvrtcCompileProgram", &a.compile) && sym(h, "nvrtcGetLoweredName", &a.lowered) &&
         sym(h, "nvrtcGetCUBINSize", &a.cubin_size) && sym(h, "nvrtcGetCUBIN", &a.cubin) &&
         sym(h, "nvrtcGetProgramLogSize", &a.log_size) && sym(h, "nvrtcGetProgramLog", &a.log) &&
         sym(h, "nvrtcDestroyProgram", &a.destroy);
  return a.ok;
}

inline bool load_driver() {
  Api& a = api();
  if (a.launch) return true;
  return drv("cuModuleLoadData", &a.module_load) && drv("cuModuleGetFunction", &a.get_function) &&
         drv("cuFuncSetAttribute", &a.set_attr) && drv("cuFuncGetAttribute", &a.get_attr) &&
         drv("cuLaunchKernelEx", &a.launch);
}

// Compile `source` (which includes the embedded headers) for sm_100a with `defines`, return the
// cubin and the lowered name of `name_expr`.  Empty cubin on failure (log in `err`).
inline bool compile(const char* source, int nheaders, const char* const* header_src, const char* const* header_names,
                    const std::string& name_expr, const std::vector<std::string>& defines, std::vector<char>* cubin,
                    std::string* lowered, std::string* err) {
  Api& a = api();
  void* prog = nullptr;
  if (a.create(&prog, source, "fg_jit.cu", nheaders, header_src, header_names) != 0) return false;
  bool ok = a.add_name(prog, name_expr.c_str()) == 0;
  std::vector<std::string> opts = {"--gpu-architecture=sm_100a", "-std=c++17", "-lineinfo",
                                   "-I" + a.include_dir};
  for (const std::string& d : defines) opts.push_back("-D" + d);
  std::vector<const char*> o;
  for (const std::string& s : opts) o.push_back(s.c_str());
  if (ok && a.compile(prog, static_cast<int>(o.size()), o.data()) != 0) {
    size_t n = 0;
    a.log_size(prog, &n);
    std::string log(n, '\0');
    if (n) a.log(prog, &log[0]);
    *err = log;
    ok = false;
  }
  if (ok) {
    const char* nm = nullptr;
    size_t n = 0;
    ok = a.lowered(prog, name_expr.c_str(), &nm) == 0 && nm && a.cubin_size(prog, &n) == 0 && n > 0;
    if (ok) {
      *lowered = nm;
      cubin->resize(n);
      ok = a.cubin(prog, cubin->data()) == 0;
    }
  }
  a.destroy(&prog);
  return ok;
}

}  // namespace fgjit
