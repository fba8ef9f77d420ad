"""Thin Python binding of the fused MoE layer: argument marshalling only.

Every step of the forward pass runs in libmoe_b200.so; torch supplies device
memory and streams.
"""

from __future__ import annotations

import ctypes

import torch

from ._lib import load_library, status_string

BF16, FP8, FP8_E5M2, MIXED = 0, 1, 2, 3
_DTYPES = {"bf16": BF16, "fp8": FP8, "e4m3": FP8, "fp8_e5m2": FP8_E5M2, "e5m2": FP8_E5M2, "mixed": MIXED,
           BF16: BF16, FP8: FP8, FP8_E5M2: FP8_E5M2, MIXED: MIXED}


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {status_string(code)} ({code})")
        self.code = code


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


class MoELayer:
    """One fused MoE layer: E experts, top-k routing, hidden H, expert intermediate I."""

    def __init__(self, E: int, topk: int, H: int, I: int, dtype="bf16"):
        self.lib = load_library()
        self.E, self.k, self.H, self.I = E, topk, H, I
        self.dtype = _DTYPES[dtype]
        h = ctypes.c_void_p()
        self._check("moe_create", self.lib.moe_create(E, topk, H, I, self.dtype, ctypes.byref(h)))
        self.handle = h.value

    def _check(self, fn, code):
        if code != 0:
            raise MoEError(fn, code)

    def _check_weights(self, fn, tensors, I_rows: int, dtype):
        """W_gate [E, I_rows, H], W_up [E, I_rows, H], W_down [E, H, I_rows], contiguous, of
        `dtype`, in device memory (the load kernels read them through raw pointers)."""
        shapes = ((self.E, I_rows, self.H), (self.E, I_rows, self.H), (self.E, self.H, I_rows))
        for name, t, shape in zip(("w_gate", "w_up", "w_down"), tensors, shapes):
            if (not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != dtype or tuple(t.shape) != shape
                    or not t.is_contiguous()):
                got = f"{t.dtype} {tuple(t.shape)} on {t.device}" if isinstance(t, torch.Tensor) else type(t).__name__
                raise ValueError(f"{fn}: {name} must be a contiguous {dtype} {list(shape)} device tensor (got {got})")

    def _check_tokens(self, fn, x, logits, out, on_gpu: bool):
        """The library takes raw pointers and trusts their sizes: reject tensors whose
        shape, dtype, layout or device would make it read or write outside them."""
        bad = []
        M = x.shape[0] if x.dim() == 2 else -1
        if x.dim() != 2 or x.shape[1] != self.H or x.dtype != torch.bfloat16 or not x.is_contiguous():
            bad.append(f"x must be a contiguous bf16 [M, {self.H}] tensor (got {x.dtype} {tuple(x.shape)})")
        if tuple(logits.shape) != (M, self.E) or logits.dtype != torch.float32 or not logits.is_contiguous():
            bad.append(f"logits must be a contiguous fp32 [{M}, {self.E}] tensor (got {logits.dtype} "
                       f"{tuple(logits.shape)})")
        if tuple(out.shape) != (M, self.H) or out.dtype != torch.bfloat16 or not out.is_contiguous():
            bad.append(f"out must be a contiguous bf16 [{M}, {self.H}] tensor (got {out.dtype} {tuple(out.shape)})")
        for name, t in (("x", x), ("logits", logits), ("out", out)):
            if t.is_cuda != on_gpu:
                bad.append(f"{name} must be in {'device' if on_gpu else 'host'} memory")
        if bad:
            raise ValueError(f"{fn}: " + "; ".join(bad))

    @property
    def is_fp8(self) -> bool:
        return self.dtype in (FP8, FP8_E5M2)

    def close(self):
        if getattr(self, "handle", None):
            self.lib.moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ weights
    def load_weights(self, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, stream=None):
        """bf16 device tensors W_gate [E,I,H], W_up [E,I,H], W_down [E,H,I]."""
        self._check_weights("moe_load_weights", (w_gate, w_up, w_down), self.I, torch.bfloat16)
        self._check("moe_load_weights", self.lib.moe_load_weights(
            self.handle, _ptr(w_gate), _ptr(w_up), _ptr(w_down), _stream(stream)))

    def load_weights_mixed(self, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, expert_fp8,
                           stream=None):
        """A "mixed" layer: bf16 device tensors as for load_weights, and expert_fp8 [E]
        booleans (host) choosing e4m3 (True) or bf16 (False) per expert."""
        self._check_weights("moe_load_weights_mixed", (w_gate, w_up, w_down), self.I, torch.bfloat16)
        flags = torch.as_tensor([1 if f else 0 for f in expert_fp8], dtype=torch.uint8)
        if flags.numel() != self.E:
            raise ValueError(f"moe_load_weights_mixed: expert_fp8 must hold {self.E} flags (got {flags.numel()})")
        self._check("moe_load_weights_mixed", self.lib.moe_load_weights_mixed(
            self.handle, _ptr(w_gate), _ptr(w_up), _ptr(w_down), flags.data_ptr(), _stream(stream)))

    def load_weights_shard(self, w_gate: torch.Tensor, w_up: torch.Tensor, w_down: torch.Tensor, shard: int,
                           num_shards: int, stream=None):
        """Shard `shard` of `num_shards` over the intermediate dimension, from the FULL bf16
        device tensors W_gate [E,I_full,H], W_up [E,I_full,H], W_down [E,H,I_full]
        (I_full = I * num_shards); the slicing happens in the library's load kernels."""
        I_full = self.I * num_shards
        self._check_weights("moe_load_weights_shard", (w_gate, w_up, w_down), I_full, torch.bfloat16)
        self._check("moe_load_weights_shard", self.lib.moe_load_weights_shard(
            self.handle, _ptr(w_gate), _ptr(w_up), _ptr(w_down), I_full, shard, num_shards, _stream(stream)))

    def load_weights_fp8(self, q_gate, q_up, q_down, scales, stream=None):
        """uint8 e4m3 codes (device) and scales [E,3] fp32 (host)."""
        self._check_weights("moe_load_weights_fp8", (q_gate, q_up, q_down), self.I, torch.uint8)
        sc = torch.as_tensor(scales, dtype=torch.float32).contiguous().cpu()
        if tuple(sc.shape) != (self.E, 3):
            raise ValueError(f"moe_load_weights_fp8: scales must be [{self.E}, 3] (got {tuple(sc.shape)})")
        self._check("moe_load_weights_fp8", self.lib.moe_load_weights_fp8(
            self.handle, _ptr(q_gate), _ptr(q_up), _ptr(q_down), sc.data_ptr(), _stream(stream)))

    def reserve(self, M_max: int, stream=None):
        self._check("moe_reserve", self.lib.moe_reserve(self.handle, M_max, _stream(stream)))

    # ------------------------------------------------------------------ forward
    def forward(self, x: torch.Tensor, logits: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        M = x.shape[0]
        if out is None:
            out = torch.empty((M, self.H), dtype=torch.bfloat16, device=x.device)
        self._check_tokens("moe_forward", x, logits, out, on_gpu=True)
        self._check("moe_forward", self.lib.moe_forward(
            self.handle, _ptr(x), _ptr(logits), M, _ptr(out), _stream(stream)))
        return out

    __call__ = forward

    def forward_noalloc(self, x: torch.Tensor, logits: torch.Tensor, out: torch.Tensor, stream=None):
        """moe_forward_noalloc: the same forward with all per-call scratch taken from the
        library's fixed 32 MiB device array (no allocation inside the call)."""
        self._check_tokens("moe_forward_noalloc", x, logits, out, on_gpu=True)
        self._check("moe_forward_noalloc", self.lib.moe_forward_noalloc(
            self.handle, _ptr(x), _ptr(logits), x.shape[0], _ptr(out), _stream(stream)))
        return out

    def forward_raw(self, x_ptr: int, logits_ptr: int, M: int, out_ptr: int, stream_handle: int):
        self._check("moe_forward", self.lib.moe_forward(self.handle, x_ptr, logits_ptr, M, out_ptr, stream_handle))

    def forward_host(self, x_cpu: torch.Tensor, logits_cpu: torch.Tensor, out_cpu: torch.Tensor, stream=None):
        M = x_cpu.shape[0]
        self._check_tokens("moe_forward_host", x_cpu, logits_cpu, out_cpu, on_gpu=False)
        self._check("moe_forward_host", self.lib.moe_forward_host(
            self.handle, _ptr(x_cpu), _ptr(logits_cpu), M, _ptr(out_cpu), _stream(stream)))
        return out_cpu

    def set_fused_decode(self, enable: bool = True):
        """Single-launch decode path (bf16, M <= 64) instead of the kernel chain."""
        self._check("moe_set_fused_decode", self.lib.moe_set_fused_decode(self.handle, 1 if enable else 0))

    def set_gemv_max_tokens(self, max_tokens: int):
        """Largest batch run on the thin-batch path (warp-level tensor-core products); 0 = never, -1 = default."""
        self._check("moe_set_gemv_max_tokens", self.lib.moe_set_gemv_max_tokens(self.handle, int(max_tokens)))

    @property
    def last_launch_count(self) -> int:
        return self.lib.moe_last_launch_count(self.handle)

    @property
    def last_gemm_pairs(self) -> bool:
        """Whether the last forward's grouped GEMMs ran on CTA pairs."""
        return self.lib.moe_last_gemm_pairs(self.handle) == 1

    KERNEL_SLOTS = ("route", "align", "gather", "gate_up", "quant_h", "down", "finalize")

    def profile_enable(self, enable: bool = True):
        self._check("moe_profile_enable", self.lib.moe_profile_enable(self.handle, 1 if enable else 0))

    def profile_read(self):
        """{kernel: (total ms, launches)} since profiling was enabled."""
        ms = (ctypes.c_double * 7)()
        n = (ctypes.c_int * 7)()
        self._check("moe_profile_read", self.lib.moe_profile_read(self.handle, ctypes.addressof(ms),
                                                                  ctypes.addressof(n)))
        return {k: (ms[i], n[i]) for i, k in enumerate(self.KERNEL_SLOTS)}

    def device_error(self) -> int:
        """The device error word (0 = no kernel reported an error); reading clears it."""
        c = ctypes.c_int(0)
        rc = self.lib.moe_get_device_error(self.handle, ctypes.byref(c))
        if rc != 0 and c.value == 0:
            self._check("moe_get_device_error", rc)
        return c.value

    # ------------------------------------------------------------------ test access
    def debug_routing(self, M: int):
        dev = torch.device("cuda")
        P = M * self.k
        ids = torch.empty((M, self.k), dtype=torch.int32, device=dev)
        w = torch.empty((M, self.k), dtype=torch.float32, device=dev)
        counts = torch.empty(self.E, dtype=torch.int32, device=dev)
        poff = torch.empty(self.E + 1, dtype=torch.int32, device=dev)
        cap = P + min(self.E, P) * 15 + 16
        pairs = torch.empty(cap, dtype=torch.int32, device=dev)
        scales = torch.empty(2, dtype=torch.float32)
        tile = ctypes.c_int(0)
        self._check("moe_debug_routing", self.lib.moe_debug_routing(
            self.handle, _ptr(ids), _ptr(w), _ptr(counts), _ptr(poff), _ptr(pairs), scales.data_ptr(),
            ctypes.byref(tile)))
        rows = int(poff[-1].item())
        return {"ids": ids, "w": w, "counts": counts, "padded_offsets": poff, "padded_pairs": pairs[:rows],
                "s_x": float(scales[0]), "s_h": float(scales[1]), "tile_rows": tile.value}

    def debug_activations(self, rows: int):
        dev = torch.device("cuda")
        xp = torch.empty((rows, self.H), dtype=torch.uint8 if self.is_fp8 else torch.bfloat16, device=dev)
        h = torch.empty((rows, self.I), dtype=torch.bfloat16, device=dev)
        self._check("moe_debug_activations", self.lib.moe_debug_activations(self.handle, _ptr(xp), _ptr(h)))
        return xp, h

    def debug_weights(self):
        dev = torch.device("cuda")
        dt = torch.uint8 if self.is_fp8 else torch.bfloat16
        g = torch.empty((self.E, self.I, self.H), dtype=dt, device=dev)
        u = torch.empty((self.E, self.I, self.H), dtype=dt, device=dev)
        d = torch.empty((self.E, self.H, self.I), dtype=dt, device=dev)
        sc = torch.ones((self.E, 3), dtype=torch.float32)
        self._check("moe_debug_weights", self.lib.moe_debug_weights(
            self.handle, _ptr(g), _ptr(u), _ptr(d), sc.data_ptr()))
        return g, u, d, sc


def inv_rope_fp8_quant(x: torch.Tensor, positions: torch.Tensor, cos_sin: torch.Tensor, interleaved: bool = False,
                       fmt: str = "e4m3", codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
                       stream=None):
    """moe_inv_rope_fp8_quant: x [T, NH, D] bf16, positions [T] int32, cos_sin [max_pos, D]
    fp32 (device) -> (codes [T, NH, D] uint8, scales [T, NH] fp32)."""
    lib = load_library()
    if x.dim() != 3 or x.dtype != torch.bfloat16 or not x.is_contiguous():
        raise ValueError(f"moe_inv_rope_fp8_quant: x must be a contiguous bf16 [T, NH, D] tensor "
                         f"(got {x.dtype} {tuple(x.shape)})")
    T, NH, D = x.shape
    if codes is None:
        codes = torch.empty((T, NH, D), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((T, NH), dtype=torch.float32, device=x.device)
    bad = []
    if tuple(positions.shape) != (T,) or positions.dtype != torch.int32 or not positions.is_contiguous():
        bad.append(f"positions must be a contiguous int32 [{T}] tensor")
    if cos_sin.dim() != 2 or cos_sin.shape[1] != D or cos_sin.dtype != torch.float32 or not cos_sin.is_contiguous():
        bad.append(f"cos_sin must be a contiguous fp32 [max_pos, {D}] tensor")
    if tuple(codes.shape) != (T, NH, D) or codes.dtype != torch.uint8 or not codes.is_contiguous():
        bad.append(f"codes must be a contiguous uint8 [{T}, {NH}, {D}] tensor")
    if tuple(scales.shape) != (T, NH) or scales.dtype != torch.float32 or not scales.is_contiguous():
        bad.append(f"scales must be a contiguous fp32 [{T}, {NH}] tensor")
    for name, t in (("x", x), ("positions", positions), ("cos_sin", cos_sin), ("codes", codes), ("scales", scales)):
        if not t.is_cuda:
            bad.append(f"{name} must be in device memory")
    if bad:
        raise ValueError("moe_inv_rope_fp8_quant: " + "; ".join(bad))
    rc = lib.moe_inv_rope_fp8_quant(_ptr(x), _ptr(positions), _ptr(cos_sin), cos_sin.shape[0], T, NH, D,
                                    1 if interleaved else 0, _DTYPES[fmt], _ptr(codes), _ptr(scales),
                                    _stream(stream))
    if rc != 0:
        raise MoEError("moe_inv_rope_fp8_quant", rc)
    return codes, scales
