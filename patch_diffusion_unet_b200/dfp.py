"""Python binding of libdfp (include/dfp.h): argument marshalling only.

Every step of the layer runs in the library's CUDA kernels; this module only
turns Python/torch objects into pointers and sizes.  Importing it fails loudly
when the compiled library is missing -- there is no fallback.
"""
import ctypes
import os

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdfp.so")

OK, E_ARG, E_STATE, E_CUDA, E_NOMEM, E_UNSUPPORTED, E_DEVICE = range(7)
F32, BF16 = 0, 1
BLOCK_RES_ATTN, BLOCK_SDXL_STAGE, BLOCK_UNET = 0, 1, 2
GN_CORRECTED, GN_STALE_OTHERS, GN_SYNC, GN_SEPARATE = 0, 1, 2, 3
CTX_DISPLACED, CTX_NAIVE = 0, 1
FAMILY_TENSOR_CORE, FAMILY_SIMT = 0, 1

EXPORTED = ("dfp_create", "dfp_load_weights", "dfp_step", "dfp_step_host", "dfp_step_host_async",
            "dfp_synchronize", "dfp_output",
            "dfp_copy_out", "dfp_buffer_bytes", "dfp_check_device", "dfp_launches_per_step",
            "dfp_set_kernel_family", "dfp_set_attention_kv_budget", "dfp_set_profiling", "dfp_kernel_times", "dfp_destroy",
            "dfp_last_error", "dfp_group_norm_noalloc", "dfp_group_norm_noalloc_error",
            "dfp_selftest_wait_timeout", "dfp_selftest_exp2_poly", "dfp_set_launch_overlap",
            "dfp_attention_schedule_check", "dfp_step_patches", "dfp_context_buffer", "dfp_set_timestep",
            "dfp_ddim_sample")


class Config(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("W", ctypes.c_int), ("C", ctypes.c_int),
                ("n_patches", ctypes.c_int), ("gn_groups", ctypes.c_int), ("gn_eps", ctypes.c_float),
                ("heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("dtype", ctypes.c_int),
                ("block", ctypes.c_int), ("gn_mode", ctypes.c_int), ("context", ctypes.c_int),
                ("n_xformer", ctypes.c_int), ("ffn_inner", ctypes.c_int), ("ctx_len", ctypes.c_int),
                ("ctx_dim", ctypes.c_int), ("batch", ctypes.c_int)]


class Tensor(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("ptr", ctypes.c_void_p), ("on_device", ctypes.c_int),
                ("dtype", ctypes.c_int), ("ndim", ctypes.c_int),
                ("shape", ctypes.POINTER(ctypes.c_longlong))]


def load_library(path=_LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(f"libdfp.so is not built ({path}); run "
                          "`python -m patch_diffusion_unet_b200.build` first")
    lib = ctypes.CDLL(path)
    H = ctypes.c_void_p
    sig = {
        "dfp_create": ([ctypes.POINTER(Config), ctypes.c_void_p, ctypes.POINTER(H)], ctypes.c_int),
        "dfp_load_weights": ([H, ctypes.POINTER(Tensor), ctypes.c_int], ctypes.c_int),
        "dfp_step": ([H, ctypes.c_void_p, ctypes.c_int, ctypes.c_int], ctypes.c_int),
        "dfp_step_host": ([H, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int], ctypes.c_int),
        "dfp_step_host_async": ([H, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int], ctypes.c_int),
        "dfp_synchronize": ([H], ctypes.c_int),
        "dfp_output": ([H, ctypes.POINTER(ctypes.c_void_p)], ctypes.c_int),
        "dfp_copy_out": ([H, ctypes.c_char_p, ctypes.c_void_p, ctypes.c_longlong], ctypes.c_int),
        "dfp_buffer_bytes": ([H, ctypes.c_char_p, ctypes.POINTER(ctypes.c_longlong)], ctypes.c_int),
        "dfp_check_device": ([H], ctypes.c_int),
        "dfp_launches_per_step": ([H], ctypes.c_int),
        "dfp_set_kernel_family": ([H, ctypes.c_int], ctypes.c_int),
        "dfp_set_attention_kv_budget": ([H, ctypes.c_longlong], ctypes.c_int),
        "dfp_set_launch_overlap": ([H, ctypes.c_int], ctypes.c_int),
        "dfp_attention_schedule_check": ([ctypes.c_int] * 10 + [ctypes.c_longlong], ctypes.c_int),
        "dfp_step_patches": ([H, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int], ctypes.c_int),
        "dfp_set_timestep": ([H, ctypes.c_float], ctypes.c_int),
        "dfp_ddim_sample": ([H, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                             ctypes.c_float, ctypes.c_void_p], ctypes.c_int),
        "dfp_context_buffer": ([H, ctypes.c_char_p, ctypes.c_int, ctypes.POINTER(ctypes.c_void_p),
                                ctypes.POINTER(ctypes.c_longlong)], ctypes.c_int),
        "dfp_set_profiling": ([H, ctypes.c_int], ctypes.c_int),
        "dfp_kernel_times": ([H, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_char_p), ctypes.c_int],
                             ctypes.c_int),
        "dfp_destroy": ([H], ctypes.c_int),
        "dfp_group_norm_noalloc": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p], ctypes.c_int),
        "dfp_group_norm_noalloc_error": ([], ctypes.c_char_p),
        "dfp_last_error": ([H], ctypes.c_char_p),
        "dfp_selftest_wait_timeout": ([ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_longlong)],
                                      ctypes.c_int),
        "dfp_selftest_exp2_poly": ([ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                    ctypes.c_void_p], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, res
    return lib


LIB = load_library()


class DfpError(RuntimeError):
    def __init__(self, status, msg):
        super().__init__(f"dfp status {status}: {msg}")
        self.status = status


def _dtype_code(dtype):
    return {"f32": F32, "bf16": BF16}[dtype]


def _torch_dtype(code):
    return torch.bfloat16 if code == BF16 else torch.float32


def make_config(cfg, gn_mode=GN_CORRECTED, context=CTX_DISPLACED):
    c = Config()
    c.H, c.W, c.C = cfg["H"], cfg["W"], cfg["C"]
    c.n_patches, c.gn_groups, c.gn_eps = cfg["n_patches"], cfg["gn_groups"], cfg["gn_eps"]
    c.heads, c.head_dim = cfg["heads"], cfg["head_dim"]
    c.dtype = _dtype_code(cfg["dtype"])
    c.block = {"res_attn": BLOCK_RES_ATTN, "sdxl_stage": BLOCK_SDXL_STAGE, "unet": BLOCK_UNET}[cfg["block"]]
    c.gn_mode, c.context = gn_mode, context
    c.n_xformer = cfg.get("n_xformer", 0)
    c.ffn_inner = cfg.get("ffn_inner", 0)
    c.ctx_len = cfg.get("ctx_len", 0)
    c.ctx_dim = cfg.get("ctx_dim", 0)
    c.batch = cfg.get("batch", 1)
    return c


class DisplacedPatchBlock:
    """One handle of the C library: a displaced-patch layer (block) on one GPU."""

    def __init__(self, cfg, stream=None, gn_mode=GN_CORRECTED, context=CTX_DISPLACED):
        self.cfg = cfg
        self.dtype = _dtype_code(cfg["dtype"])
        self.tdtype = _torch_dtype(self.dtype)
        if stream is None:
            stream = torch.cuda.current_stream()
        self.stream = stream
        self._c = make_config(cfg, gn_mode, context)
        h = ctypes.c_void_p()
        st = LIB.dfp_create(ctypes.byref(self._c), ctypes.c_void_p(stream.cuda_stream), ctypes.byref(h))
        if st != OK:
            raise DfpError(st, LIB.dfp_last_error(None).decode())
        self.h = h

    # ------------------------------------------------------------------ helpers
    def _check(self, st):
        if st != OK:
            raise DfpError(st, LIB.dfp_last_error(self.h).decode())

    def close(self):
        if getattr(self, "h", None):
            LIB.dfp_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ API
    def load_weights(self, weights):
        """weights: name -> numpy array or torch tensor (CPU or CUDA), fp32 or bf16."""
        keep, arr = [], (Tensor * len(weights))()
        for i, (name, w) in enumerate(weights.items()):
            if isinstance(w, np.ndarray):
                w = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32))
            w = w.contiguous()
            if w.dtype not in (torch.float32, torch.bfloat16):
                w = w.float()
            shape = (ctypes.c_longlong * w.dim())(*w.shape)
            nm = name.encode()
            keep += [w, shape, nm]
            arr[i] = Tensor(nm, w.data_ptr(), int(w.is_cuda), BF16 if w.dtype == torch.bfloat16 else F32,
                            w.dim(), shape)
        self._check(LIB.dfp_load_weights(self.h, arr, len(weights)))

    def step(self, x, step, is_sync):
        """x: contiguous CUDA tensor [B, H, W, C] (B = cfg "batch", default 1; [H, W, C] for one
        image) of the config dtype (must outlive the stream work)."""
        if not (x.is_cuda and x.is_contiguous() and x.dtype == self.tdtype):
            raise ValueError("x must be a contiguous CUDA tensor of the config dtype")
        self._check(LIB.dfp_step(self.h, ctypes.c_void_p(x.data_ptr()), int(step), int(is_sync)))

    def step_host(self, x_host, y_host, step, is_sync):
        """Host-buffer step: x_host / y_host are CPU tensors (pinned for async copies)."""
        self._check(LIB.dfp_step_host(self.h, ctypes.c_void_p(x_host.data_ptr()),
                                      ctypes.c_void_p(y_host.data_ptr()), int(step), int(is_sync)))

    def step_host_async(self, x_host, y_host, step, is_sync):
        """Pipelined host-buffer step (pinned CPU tensors): returns once enqueued; x_host
        must stay unchanged and y_host is filled after synchronize()."""
        self._check(LIB.dfp_step_host_async(self.h, ctypes.c_void_p(x_host.data_ptr()),
                                            ctypes.c_void_p(y_host.data_ptr()), int(step), int(is_sync)))

    def synchronize(self):
        self._check(LIB.dfp_synchronize(self.h))

    def buffer(self, name):
        """A fresh torch copy (on the device) of an internal buffer of the last step."""
        nbytes = ctypes.c_longlong()
        self._check(LIB.dfp_buffer_bytes(self.h, name.encode(), ctypes.byref(nbytes)))
        if name.startswith("gn") or name == "lat":
            out = torch.empty(nbytes.value // 4, dtype=torch.float32, device="cuda")
        else:
            out = torch.empty(nbytes.value // (2 if self.dtype == BF16 else 4), dtype=self.tdtype, device="cuda")
        self._check(LIB.dfp_copy_out(self.h, name.encode(), ctypes.c_void_p(out.data_ptr()), nbytes.value))
        return out

    def output(self):
        cols = self.cfg["latent_c"] if self.cfg["block"] == "unet" else self.cfg["C"]
        return self.buffer("y").view(self.cfg.get("batch", 1) * self.cfg["H"] * self.cfg["W"], cols)

    def set_timestep(self, tau):
        """UNet block: the timestep the next step embeds."""
        self._check(LIB.dfp_set_timestep(self.h, float(tau)))

    def ddim_sample(self, x_T, n_steps, n_sync, n_train=1000, beta_start=0.00085, beta_end=0.012, out=None):
        """UNet block: the DDIM loop from x_T (CUDA fp32 [H, W, 4]); returns the final latent
        (asynchronous on the handle's stream)."""
        if not (x_T.is_cuda and x_T.is_contiguous() and x_T.dtype == torch.float32):
            raise ValueError("x_T must be a contiguous CUDA fp32 tensor")
        out = torch.empty_like(x_T) if out is None else out
        self._check(LIB.dfp_ddim_sample(self.h, ctypes.c_void_p(x_T.data_ptr()), int(n_steps), int(n_sync),
                                        int(n_train), float(beta_start), float(beta_end),
                                        ctypes.c_void_p(out.data_ptr())))
        return out

    def check_device(self):
        self._check(LIB.dfp_check_device(self.h))

    def launches_per_step(self):
        return LIB.dfp_launches_per_step(self.h)

    def set_profiling(self, enable=True):
        self._check(LIB.dfp_set_profiling(self.h, int(enable)))

    def kernel_times(self):
        """[(kernel name, milliseconds)] of the last profiled step."""
        ms = (ctypes.c_float * 128)()
        names = (ctypes.c_char_p * 128)()
        n = LIB.dfp_kernel_times(self.h, ms, names, 128)
        if n < 0:
            raise DfpError(E_CUDA, "kernel timing failed")
        return [(names[i].decode(), float(ms[i])) for i in range(n)]

    def set_kernel_family(self, family):
        self._check(LIB.dfp_set_kernel_family(self.h, int(family)))

    def set_attention_kv_budget(self, nbytes):
        """K/V bytes above which the attention deals whole-unit rounds (0: the kernel's own)."""
        self._check(LIB.dfp_set_attention_kv_budget(self.h, int(nbytes)))

    def set_launch_overlap(self, enable=True):
        """Programmatic dependent launch between the step's kernels (on by default)."""
        self._check(LIB.dfp_set_launch_overlap(self.h, int(enable)))
