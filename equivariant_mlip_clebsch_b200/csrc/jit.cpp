// jit.cpp -- runtime compilation of the path-specialised kernels.
//
// Each plan generates CUDA source whose loops are fully specialised to its
// paths (degrees, multiplicities, offsets, coefficient layouts), compiles it
// with NVRTC straight to an sm_100a cubin and loads it through the driver
// API.  The driver entry points are fetched from the CUDA runtime
// (cudaGetDriverEntryPoint) so the library does not link libcuda itself.
// Cubins can be cached on disk: set CGTP_JIT_CACHE to a writable directory.
#include <cuda.h>
#include <nvrtc.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <fstream>
#include <functional>
#include <sstream>
#include <thread>
#include <unistd.h>

#include "internal.hpp"

namespace cgtp {

namespace {

struct Driver {
  CUresult (*moduleLoadData)(CUmodule*, const void*) = nullptr;
  CUresult (*moduleGetFunction)(CUfunction*, CUmodule, const char*) = nullptr;
  CUresult (*moduleUnload)(CUmodule) = nullptr;
  CUresult (*funcSetAttribute)(CUfunction, CUfunction_attribute, int) = nullptr;
  CUresult (*launchKernel)(CUfunction, unsigned, unsigned, unsigned, unsigned, unsigned, unsigned,
                           unsigned, CUstream, void**, void**) = nullptr;
  CUresult (*launchKernelEx)(const CUlaunchConfig*, CUfunction, void**, void**) = nullptr;
  CUresult (*getErrorString)(CUresult, const char**) = nullptr;
  CUresult (*occupancy)(int*, CUfunction, int, size_t) = nullptr;
  bool ok = false;
  std::string err;
};

template <class F>
bool entry(const char* sym, F& fp, std::string& err) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint(sym, &p, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p) {
    err = std::string("driver entry point ") + sym + " unavailable";
    return false;
  }
  fp = reinterpret_cast<F>(p);
  return true;
}

Driver& driver() {
  static Driver d;
  static std::once_flag once;
  std::call_once(once, [] {
    std::string err;
    d.ok = entry("cuModuleLoadData", d.moduleLoadData, err) &&
           entry("cuModuleGetFunction", d.moduleGetFunction, err) &&
           entry("cuModuleUnload", d.moduleUnload, err) &&
           entry("cuFuncSetAttribute", d.funcSetAttribute, err) &&
           entry("cuLaunchKernel", d.launchKernel, err) &&
           entry("cuGetErrorString", d.getErrorString, err) &&
           entry("cuOccupancyMaxActiveBlocksPerMultiprocessor", d.occupancy, err);
    d.err = err;
    std::string ignore;  // optional: without it, launches are plain
    entry("cuLaunchKernelEx", d.launchKernelEx, ignore);
  });
  return d;
}

std::string cu_str(CUresult r) {
  const char* s = nullptr;
  if (driver().getErrorString) driver().getErrorString(r, &s);
  return s ? s : ("CUresult " + std::to_string((int)r));
}

uint64_t fnv1a(const std::string& s, uint64_t h = 1469598103934665603ull) {
  for (unsigned char c : s) {
    h ^= c;
    h *= 1099511628211ull;
  }
  return h;
}

bool read_file(const std::string& path, std::string& out) {
  std::ifstream f(path, std::ios::binary);
  if (!f) return false;
  std::ostringstream ss;
  ss << f.rdbuf();
  out = ss.str();
  return !out.empty();
}

void write_file_atomic(const std::string& path, const std::string& data) {
  std::string tmp = path + ".tmp" + std::to_string((long)::getpid()) + "_" +
                    std::to_string(std::hash<std::thread::id>()(std::this_thread::get_id()));
  {
    std::ofstream f(tmp, std::ios::binary);
    if (!f) return;
    f.write(data.data(), (std::streamsize)data.size());
  }
  std::rename(tmp.c_str(), path.c_str());
}

}  // namespace

static const char* kOpts[] = {"--gpu-architecture=sm_100a", "-std=c++17", "-lineinfo",
                              "-DNDEBUG", "--ptxas-options=-v"};

// Compile to a cubin (no device needed).  Fills k.log with the compiler and
// assembler messages (registers, spills).
static cgtp_status compile_cubin(const std::string& src, const std::string& name, std::string& cubin,
                                 std::string& log, unsigned long long& hash) {
  int maj = 0, mnr = 0;
  nvrtcVersion(&maj, &mnr);
  std::string key = src;
  for (const char* o : kOpts) key += std::string("|") + o;
  key += "|nvrtc" + std::to_string(maj) + "." + std::to_string(mnr);
  hash = fnv1a(key);
  const char* cache = std::getenv("CGTP_JIT_CACHE");
  std::string cpath;
  if (cache && *cache) {
    char hx[32];
    std::snprintf(hx, sizeof hx, "%016llx", (unsigned long long)fnv1a(key));
    cpath = std::string(cache) + "/" + name + "_" + hx + ".cubin";
    if (read_file(cpath, cubin)) {
      read_file(cpath + ".log", log);
      return CGTP_OK;
    }
  }
  nvrtcProgram prog;
  if (nvrtcCreateProgram(&prog, src.c_str(), (name + ".cu").c_str(), 0, nullptr, nullptr) !=
      NVRTC_SUCCESS)
    return fail(CGTP_ERR_JIT, "nvrtcCreateProgram failed");
  nvrtcResult r = nvrtcCompileProgram(prog, (int)(sizeof(kOpts) / sizeof(kOpts[0])), kOpts);
  size_t ls = 0;
  nvrtcGetProgramLogSize(prog, &ls);
  log.assign(ls, '\0');
  if (ls) nvrtcGetProgramLog(prog, &log[0]);
  while (!log.empty() && log.back() == '\0') log.pop_back();
  if (r != NVRTC_SUCCESS) {
    nvrtcDestroyProgram(&prog);
    return fail(CGTP_ERR_JIT, "NVRTC compilation of " + name + " failed:\n" + log);
  }
  size_t cs = 0;
  nvrtcGetCUBINSize(prog, &cs);
  cubin.assign(cs, '\0');
  nvrtcGetCUBIN(prog, &cubin[0]);
  nvrtcDestroyProgram(&prog);
  if (!cpath.empty()) {
    write_file_atomic(cpath, cubin);
    write_file_atomic(cpath + ".log", log);
  }
  return CGTP_OK;
}

cgtp_status jit_build(const std::string& src, const std::string& name, JitBinary& b) {
  const cgtp_status st = compile_cubin(src, name, b.cubin, b.log, b.hash);
  if (st != CGTP_OK) b.err = cgtp_last_error();  // this thread's message, for the caller's
  return st;
}

cgtp_status jit_compile(const std::string& src, const std::string& name, JitKernel& k) {
  JitBinary b;
  const cgtp_status st = jit_build(src, name, b);
  if (st != CGTP_OK) return st;
  return jit_load(b, name, k);
}

cgtp_status jit_load(const JitBinary& b, const std::string& name, JitKernel& k) {
  k.log = b.log;
  k.hash = b.hash;
  k.name = name;
  if (std::getenv("CGTP_JIT_COMPILE_ONLY")) return CGTP_OK;  // host-only checks
  Driver& d = driver();
  if (!d.ok) return fail(CGTP_ERR_CUDA, d.err);
  CUmodule mod;
  CUresult cr = d.moduleLoadData(&mod, b.cubin.data());
  if (cr != CUDA_SUCCESS) return fail(CGTP_ERR_CUDA, "cuModuleLoadData: " + cu_str(cr));
  CUfunction fn;
  cr = d.moduleGetFunction(&fn, mod, name.c_str());
  if (cr != CUDA_SUCCESS) {
    d.moduleUnload(mod);
    return fail(CGTP_ERR_CUDA, "cuModuleGetFunction: " + cu_str(cr));
  }
  if (k.smem > 48 * 1024) {
    cr = d.funcSetAttribute(fn, CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES, k.smem);
    if (cr != CUDA_SUCCESS) {
      d.moduleUnload(mod);
      return fail(CGTP_ERR_CUDA, "cuFuncSetAttribute(smem): " + cu_str(cr));
    }
  }
  int nb = 0;
  cr = d.occupancy(&nb, fn, k.threads, (size_t)k.smem);
  if (cr != CUDA_SUCCESS || nb < 1) {
    d.moduleUnload(mod);
    return fail(CGTP_ERR_CUDA, "kernel " + name + " cannot be resident: " + cu_str(cr));
  }
  k.blocks_per_sm = nb;
  k.module = mod;
  k.function = fn;
  return CGTP_OK;
}

cgtp_status jit_launch(const JitKernel& k, dim3 grid, void** args, cudaStream_t stream) {
  if (!k.function) return fail(CGTP_ERR_CUDA, "kernel " + k.name + " is not loaded");
  Driver& d = driver();
  CUresult cr;
  if (d.launchKernelEx) {
    // programmatic dependent launch: the kernel may start while its
    // predecessor on the stream finishes; it waits (griddepcontrol.wait)
    // before touching any memory the predecessor writes
    CUlaunchAttribute attr[1];
    attr[0].id = CU_LAUNCH_ATTRIBUTE_PROGRAMMATIC_STREAM_SERIALIZATION;
    attr[0].value.programmaticStreamSerializationAllowed = 1;
    CUlaunchConfig cfg = {};
    cfg.gridDimX = grid.x;
    cfg.gridDimY = grid.y;
    cfg.gridDimZ = grid.z;
    cfg.blockDimX = (unsigned)k.threads;
    cfg.blockDimY = 1;
    cfg.blockDimZ = 1;
    cfg.sharedMemBytes = (unsigned)k.smem;
    cfg.hStream = (CUstream)stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cr = d.launchKernelEx(&cfg, (CUfunction)k.function, args, nullptr);
  } else {
    cr = d.launchKernel((CUfunction)k.function, grid.x, grid.y, grid.z, k.threads, 1, 1, k.smem,
                        (CUstream)stream, args, nullptr);
  }
  if (cr != CUDA_SUCCESS) return fail(CGTP_ERR_CUDA, "launch of " + k.name + ": " + cu_str(cr));
  return CGTP_OK;
}

void jit_unload(JitKernel& k) {
  if (k.module && driver().ok) driver().moduleUnload((CUmodule)k.module);
  k.module = nullptr;
  k.function = nullptr;
}

}  // namespace cgtp
