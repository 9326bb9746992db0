// jit.cu -- runtime specialisation of the tile GEMM kernel (opt-in, FG_JIT=1).
//
// The pages' library compiles its kernels at run time for each shape (a
// lightweight JIT; chujupifa.com "机器之心报道", opening summary) and keeps
// them in an on-disk cache (deepseek.csdn.net "DeepGEMM：简洁、高效…", section
// "环境变量": a cache directory and the compiler to use).  Here the kernel
// headers of this library are compiled with NVRTC for one (block width, CTA
// pair, K blocks) triple, the K block count becoming a compile-time constant
// of the kernel (FG8_KB_CT), for sm_100a.  The cubin is cached under
// FG_CACHE_DIR (default $HOME/.cache/fg8) by a hash of the kernel sources, the
// options and the specialisation; later processes load it from there.  NVRTC
// is opened at run time (dlopen), so the library needs it only when the JIT is
// used; any failure leaves the ahead-of-time kernels in use.
#include <cuda.h>
#include <cuda_runtime.h>
#include <dlfcn.h>
#include <sys/stat.h>
#include <unistd.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <tuple>
#include <vector>

#include "fg8.h"
#include "jit.h"
#include "launch.cuh"

namespace fg8 {
namespace {

// ---- NVRTC, opened at run time ----------------------------------------------
typedef struct _nvrtcProgram* nvrtcProgram;
typedef int nvrtcResult;
struct Nvrtc {
    bool ok = false;
    nvrtcResult (*create)(nvrtcProgram*, const char*, const char*, int, const char* const*, const char* const*);
    nvrtcResult (*compile)(nvrtcProgram, int, const char* const*);
    nvrtcResult (*log_size)(nvrtcProgram, size_t*);
    nvrtcResult (*log)(nvrtcProgram, char*);
    nvrtcResult (*cubin_size)(nvrtcProgram, size_t*);
    nvrtcResult (*cubin)(nvrtcProgram, char*);
    nvrtcResult (*add_name)(nvrtcProgram, const char*);
    nvrtcResult (*lowered)(nvrtcProgram, const char*, const char**);
    nvrtcResult (*destroy)(nvrtcProgram*);
};

const Nvrtc& nvrtc() {
    static Nvrtc n = [] {
        Nvrtc r;
        const char* names[] = {"libnvrtc.so.12", "libnvrtc.so", "/usr/local/cuda/lib64/libnvrtc.so.12"};
        void* h = nullptr;
        for (const char* nm : names)
            if ((h = dlopen(nm, RTLD_NOW | RTLD_LOCAL)) != nullptr) break;
        if (!h) return r;
#define FG8_SYM(field, name) r.field = reinterpret_cast<decltype(r.field)>(dlsym(h, name))
        FG8_SYM(create, "nvrtcCreateProgram");
        FG8_SYM(compile, "nvrtcCompileProgram");
        FG8_SYM(log_size, "nvrtcGetProgramLogSize");
        FG8_SYM(log, "nvrtcGetProgramLog");
        FG8_SYM(cubin_size, "nvrtcGetCUBINSize");
        FG8_SYM(cubin, "nvrtcGetCUBIN");
        FG8_SYM(add_name, "nvrtcAddNameExpression");
        FG8_SYM(lowered, "nvrtcGetLoweredName");
        FG8_SYM(destroy, "nvrtcDestroyProgram");
#undef FG8_SYM
        r.ok = r.create && r.compile && r.log_size && r.log && r.cubin_size && r.cubin && r.add_name && r.lowered &&
               r.destroy;
        return r;
    }();
    return n;
}

// ---- driver entry points ------------------------------------------------------
struct Driver {
    bool ok = false;
    CUresult (*module_load)(CUmodule*, const void*);
    CUresult (*get_function)(CUfunction*, CUmodule, const char*);
    CUresult (*func_get_attr)(int*, CUfunction_attribute, CUfunction);
    CUresult (*func_set_attr)(CUfunction, CUfunction_attribute, int);
    CUresult (*launch_ex)(const CUlaunchConfig*, CUfunction, void**, void**);
};

const Driver& driver() {
    static Driver d = [] {
        Driver r;
        auto get = [](const char* name) -> void* {
            void* p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
                q != cudaDriverEntryPointSuccess) {
                cudaGetLastError();
                return nullptr;
            }
            return p;
        };
        r.module_load = reinterpret_cast<decltype(r.module_load)>(get("cuModuleLoadData"));
        r.get_function = reinterpret_cast<decltype(r.get_function)>(get("cuModuleGetFunction"));
        r.func_get_attr = reinterpret_cast<decltype(r.func_get_attr)>(get("cuFuncGetAttribute"));
        r.func_set_attr = reinterpret_cast<decltype(r.func_set_attr)>(get("cuFuncSetAttribute"));
        r.launch_ex = reinterpret_cast<decltype(r.launch_ex)>(get("cuLaunchKernelEx"));
        r.ok = r.module_load && r.get_function && r.func_get_attr && r.func_set_attr && r.launch_ex;
        return r;
    }();
    return d;
}

// ---- sources -----------------------------------------------------------------
// The kernel headers next to this library (<library dir>/csrc), read once.
std::string csrc_dir() {
    Dl_info info;
    if (dladdr(reinterpret_cast<void*>(&fg_version), &info) && info.dli_fname) {
        std::string p(info.dli_fname);
        const size_t slash = p.rfind('/');
        return (slash == std::string::npos ? std::string(".") : p.substr(0, slash)) + "/csrc";
    }
    return "csrc";
}

bool read_file(const std::string& path, std::string* out) {
    FILE* f = std::fopen(path.c_str(), "rb");
    if (!f) return false;
    std::string s;
    char buf[65536];
    size_t n;
    while ((n = std::fread(buf, 1, sizeof(buf), f)) > 0) s.append(buf, n);
    std::fclose(f);
    *out = s;
    return true;
}

struct Sources {
    bool ok = false;
    std::vector<std::string> names, texts;
};

const Sources& sources() {
    static Sources s = [] {
        Sources r;
        const std::string dir = csrc_dir();
        for (const char* nm : {"gemm_kernel.cuh", "ptx.cuh", "rtc_compat.cuh"}) {
            std::string t;
            if (!read_file(dir + "/" + nm, &t)) return r;
            r.names.push_back(nm);
            r.texts.push_back(t);
        }
        r.ok = true;
        return r;
    }();
    return s;
}

std::string cuda_include_dir() {
    const char* e = std::getenv("CUDA_HOME");
    std::string base = e ? e : "/usr/local/cuda";
    return base + "/include";
}

uint64_t fnv1a(const std::string& s, uint64_t h = 1469598103934665603ull) {
    for (unsigned char c : s) {
        h ^= c;
        h *= 1099511628211ull;
    }
    return h;
}

std::string cache_dir() {
    const char* e = std::getenv("FG_CACHE_DIR");
    if (e && *e) return e;
    const char* home = std::getenv("HOME");
    return std::string(home ? home : "/tmp") + "/.cache/fg8";
}

void make_dirs(const std::string& path) {
    std::string cur;
    for (size_t i = 0; i < path.size(); ++i) {
        cur += path[i];
        if (path[i] == '/' && cur.size() > 1) mkdir(cur.c_str(), 0755);
    }
    mkdir(path.c_str(), 0755);
}

std::atomic<int> g_compiled{0}, g_from_disk{0}, g_launches{0};

struct Spec {
    int bn, pair, kb;
};

// The cubin of one specialisation: from the disk cache, else compiled now and
// written there.  Returns the lowered kernel name in *name.
fg_status get_cubin(const Spec& sp, std::string* cubin, std::string* name, std::string* path_out) {
    const Sources& src = sources();
    if (!src.ok) return FG_ERR_UNSUPPORTED;
    char expr[96];
    std::snprintf(expr, sizeof(expr), "fg8::fg8_gemm_kernel<%d, %s>", sp.bn, sp.pair ? "true" : "false");
    char def[64];
    std::snprintf(def, sizeof(def), "-DFG8_KB_CT=%d", sp.kb);
    const std::string inc = "-I" + cuda_include_dir();
    const std::vector<std::string> opts = {"--gpu-architecture=sm_100a", "-std=c++17", "-default-device", def, inc};
    const std::string program = "#include \"gemm_kernel.cuh\"\n";
    uint64_t h = fnv1a(program);
    for (const auto& t : src.texts) h = fnv1a(t, h);
    for (const auto& o : opts) h = fnv1a(o, h);
    h = fnv1a(expr, h);
    char fname[64];
    std::snprintf(fname, sizeof(fname), "/fg8_%016llx.cubin", static_cast<unsigned long long>(h));
    const std::string dir = cache_dir();
    const std::string path = dir + fname;
    const std::string name_path = path + ".name";
    if (path_out) *path_out = path;
    if (read_file(path, cubin) && read_file(name_path, name) && !cubin->empty() && !name->empty()) {
        g_from_disk.fetch_add(1);
        return FG_OK;
    }
    const Nvrtc& nv = nvrtc();
    if (!nv.ok) return FG_ERR_UNSUPPORTED;
    std::vector<const char*> hdr_names, hdr_texts;
    for (size_t i = 0; i < src.names.size(); ++i) {
        hdr_names.push_back(src.names[i].c_str());
        hdr_texts.push_back(src.texts[i].c_str());
    }
    nvrtcProgram prog = nullptr;
    if (nv.create(&prog, program.c_str(), "fg8_jit.cu", static_cast<int>(hdr_names.size()), hdr_texts.data(),
                  hdr_names.data()) != 0)
        return FG_ERR_CUDA;
    nv.add_name(prog, expr);
    std::vector<const char*> o;
    for (const auto& s : opts) o.push_back(s.c_str());
    const nvrtcResult rc = nv.compile(prog, static_cast<int>(o.size()), o.data());
    if (rc != 0) {
        if (std::getenv("FG_JIT_VERBOSE")) {
            size_t n = 0;
            nv.log_size(prog, &n);
            std::string log(n, '\0');
            nv.log(prog, &log[0]);
            std::fprintf(stderr, "fg8 jit: compilation failed:\n%s\n", log.c_str());
        }
        nv.destroy(&prog);
        return FG_ERR_CUDA;
    }
    size_t n = 0;
    const char* lowered = nullptr;
    if (nv.cubin_size(prog, &n) != 0 || nv.lowered(prog, expr, &lowered) != 0 || !lowered) {
        nv.destroy(&prog);
        return FG_ERR_CUDA;
    }
    cubin->assign(n, '\0');
    nv.cubin(prog, &(*cubin)[0]);
    *name = lowered;
    nv.destroy(&prog);
    g_compiled.fetch_add(1);
    // Written to a temporary file and renamed, so a concurrent reader sees
    // either nothing or the whole file.
    make_dirs(dir);
    char tmp_suffix[32];
    std::snprintf(tmp_suffix, sizeof(tmp_suffix), ".tmp%d", static_cast<int>(getpid()));
    auto write_atomic = [&](const std::string& p, const std::string& data) {
        const std::string tmp = p + tmp_suffix;
        FILE* f = std::fopen(tmp.c_str(), "wb");
        if (!f) return;
        const bool ok = std::fwrite(data.data(), 1, data.size(), f) == data.size();
        std::fclose(f);
        if (ok) std::rename(tmp.c_str(), p.c_str());
        else std::remove(tmp.c_str());
    };
    write_atomic(name_path, *name);
    write_atomic(path, *cubin);
    return FG_OK;
}

struct Loaded {
    CUfunction fn = nullptr;
    int static_smem = 0;
};
std::map<std::tuple<int, int, int, int>, Loaded> g_loaded;   // (device, bn, pair, kb)
std::mutex g_jit_mutex;

}  // namespace

bool jit_enabled() {
    const char* e = std::getenv("FG_JIT");
    return e && std::atoi(e) == 1;
}

fg_status jit_launch_gemm(int bn, bool pair, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& td,
                          const GemmParams& p, int grid, size_t smem, cudaStream_t stream) {
    const Driver& drv = driver();
    if (!drv.ok) return FG_ERR_UNSUPPORTED;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return FG_ERR_CUDA;
    }
    Loaded L;
    {
        std::lock_guard<std::mutex> lk(g_jit_mutex);
        const auto key = std::make_tuple(dev, bn, pair ? 1 : 0, p.KB);
        auto it = g_loaded.find(key);
        if (it == g_loaded.end()) {
            std::string cubin, name;
            fg_status st = get_cubin(Spec{bn, pair ? 1 : 0, p.KB}, &cubin, &name, nullptr);
            if (st != FG_OK) return st;
            // Makes the runtime's primary context current on this thread for
            // the driver calls below (no memory is allocated).
            if (cudaFree(nullptr) != cudaSuccess) {
                cudaGetLastError();
                return FG_ERR_CUDA;
            }
            CUmodule mod = nullptr;
            if (drv.module_load(&mod, cubin.data()) != CUDA_SUCCESS) return FG_ERR_CUDA;
            CUfunction fn = nullptr;
            if (drv.get_function(&fn, mod, name.c_str()) != CUDA_SUCCESS) return FG_ERR_CUDA;
            int regs = 0, ssmem = 0;
            drv.func_get_attr(&regs, CU_FUNC_ATTRIBUTE_NUM_REGS, fn);
            drv.func_get_attr(&ssmem, CU_FUNC_ATTRIBUTE_SHARED_SIZE_BYTES, fn);
            // The in-kernel register split is safe only at exactly REGS_LAUNCH.
            if (regs != REGS_LAUNCH || ssmem > kGemmStaticSmem) return FG_ERR_UNSUPPORTED;
            if (drv.func_set_attr(fn, CU_FUNC_ATTRIBUTE_MAX_DYNAMIC_SHARED_SIZE_BYTES, kMaxDynamicSmem - ssmem) !=
                CUDA_SUCCESS)
                return FG_ERR_CUDA;
            L.fn = fn;
            L.static_smem = ssmem;
            g_loaded[key] = L;
        } else {
            L = it->second;
        }
    }
    CUlaunchConfig cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDimX = static_cast<unsigned>(grid);
    cfg.gridDimY = 1;
    cfg.gridDimZ = 1;
    cfg.blockDimX = NUM_THREADS;
    cfg.blockDimY = 1;
    cfg.blockDimZ = 1;
    cfg.sharedMemBytes = static_cast<unsigned>(smem);
    cfg.hStream = reinterpret_cast<CUstream>(stream);
    CUlaunchAttribute attr[2];
    cfg.attrs = attr;
    cfg.numAttrs = 0;
    if (pdl_enabled()) {
        attr[cfg.numAttrs].id = CU_LAUNCH_ATTRIBUTE_PROGRAMMATIC_STREAM_SERIALIZATION;
        attr[cfg.numAttrs].value.programmaticStreamSerializationAllowed = 1;
        ++cfg.numAttrs;
    }
    if (pair) {
        attr[cfg.numAttrs].id = CU_LAUNCH_ATTRIBUTE_CLUSTER_DIMENSION;
        attr[cfg.numAttrs].value.clusterDim.x = 2;
        attr[cfg.numAttrs].value.clusterDim.y = 1;
        attr[cfg.numAttrs].value.clusterDim.z = 1;
        ++cfg.numAttrs;
    }
    CUtensorMap a = ta, b = tb, d = td;
    GemmParams pp = p;
    void* args[] = {&a, &b, &d, &pp};
    if (drv.launch_ex(&cfg, L.fn, args, nullptr) != CUDA_SUCCESS) return FG_ERR_CUDA;
    g_launches.fetch_add(1);
    return FG_OK;
}

}  // namespace fg8

extern "C" fg_status fg_jit_compile(int block_n, int pair, int k_blocks, char* path_out, size_t path_len) {
    if (block_n < 16 || block_n > 256 || block_n % 16 != 0 || k_blocks <= 0 || (pair && block_n < 32))
        return FG_ERR_INVALID_ARG;
    std::string cubin, name, path;
    const fg_status st = fg8::get_cubin(fg8::Spec{block_n, pair ? 1 : 0, k_blocks}, &cubin, &name, &path);
    if (st == FG_OK && path_out && path_len > 0) {
        std::strncpy(path_out, path.c_str(), path_len - 1);
        path_out[path_len - 1] = '\0';
    }
    return st;
}

extern "C" void fg_jit_stats(int* compiled, int* loaded_from_disk, int* launches) {
    if (compiled) *compiled = fg8::g_compiled.load();
    if (loaded_from_disk) *loaded_from_disk = fg8::g_from_disk.load();
    if (launches) *launches = fg8::g_launches.load();
}
