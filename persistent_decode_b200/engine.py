"""Python handle over the C ABI: argument marshalling only.

Every step of the decode runs in libxlpk.so's kernels; torch is used here only
to hold device memory and to name the CUDA stream.
"""
from __future__ import annotations

import ctypes as C
from typing import Dict, Optional

from . import _abi

_LIB = None


def get_lib():
    """The loaded libxlpk.so (raises ImportError if it has not been built)."""
    global _LIB
    if _LIB is None:
        _LIB = _abi.load()
    return _LIB


class _LazyLib:
    def __getattr__(self, name):
        return getattr(get_lib(), name)


lib = _LazyLib()


class XlpkError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = lib.xlpk_status_string(status).decode()
        detail = lib.xlpk_last_cuda_error().decode()
        super().__init__(f"{what}: {msg}" + (f" ({detail})" if detail else ""))
        self.status = status


def _check(status: int, what: str) -> None:
    if status != _abi.XLPK_OK:
        raise XlpkError(status, what)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def tc_gemm_tile(w, x, stream=None):
    """xlpk_tc_gemm_tile: Y[N][8] = W[N][K] . X[8][K]^T on the tcgen05 tensor cores.

    `w` bf16 [N][K] and `x` fp32 [8][K] (contiguous, on the device); returns
    fp32 [N][8].  The activations enter the MMA rounded to bf16."""
    import torch
    n, k = int(w.shape[0]), int(w.shape[1])
    y = torch.empty(n, 8, dtype=torch.float32, device=w.device)
    _check(lib.xlpk_tc_gemm_tile(_ptr(w), n, k, _ptr(x), _ptr(y), _stream_handle(stream)), "xlpk_tc_gemm_tile")
    return y


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) or None


def make_config(cfg, n_ctas: int = 0, spin_limit_us: int = 0, batch: Optional[int] = None,
                max_seq: Optional[int] = None, flags: int = 0, window: int = 0) -> _abi.xlpk_config:
    c = _abi.xlpk_config()
    for f in ("n_layers", "hidden", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
              "n_experts", "top_k", "n_shared_experts", "expert_ffn"):
        setattr(c, f, int(getattr(cfg, f)))
    c.weight_dtype = {"fp8_e4m3": _abi.XLPK_DTYPE_FP8_E4M3, "nvfp4": _abi.XLPK_DTYPE_NVFP4}.get(
        cfg.weight_dtype, _abi.XLPK_DTYPE_BF16)
    c.batch = int(batch if batch is not None else cfg.batch)
    c.max_seq = int(max_seq if max_seq is not None else cfg.max_seq)
    c.rope_theta = float(cfg.rope_theta)
    c.rms_eps = float(cfg.rms_eps)
    c.n_ctas = int(n_ctas)
    c.spin_limit_us = int(spin_limit_us)
    c.flags = int(flags)
    c.window = int(window)
    if getattr(cfg, "kv_dtype", "bf16") == "fp8_e4m3":
        c.kv_dtype = _abi.XLPK_DTYPE_FP8_E4M3
        c.k_scale = float(cfg.k_scale)
        c.v_scale = float(cfg.v_scale)
    else:
        c.kv_dtype = _abi.XLPK_DTYPE_BF16
    return c


class Engine:
    """One xlpk handle.

    `weights` maps names ("embed", "lm_head", "final_norm", "layers.{l}.wq", ...,
    with ".scale" companions for FP8) to CUDA tensors in row-major [out][in]
    layout; `k_cache`/`v_cache` are CUDA tensors [L][B][n_kv][max_seq][d] (bf16,
    or uint8 e4m3 codes when cfg.kv_dtype is "fp8_e4m3") that the engine writes
    in place.  `flags` (XLPK_FLAG_*) and `window` are the
    config fields of the same names.
    """

    def __init__(self, cfg, weights: Dict[str, "object"], k_cache, v_cache, n_ctas: int = 0,
                 spin_limit_us: int = 0, flags: int = 0, window: int = 0, page_table=None,
                 max_seq: Optional[int] = None):
        self.cfg = cfg
        import torch
        want = torch.uint8 if getattr(cfg, "kv_dtype", "bf16") == "fp8_e4m3" else torch.bfloat16
        if k_cache.dtype != want or v_cache.dtype != want:
            raise ValueError(f"KV cache must be {want} for kv_dtype {getattr(cfg, 'kv_dtype', 'bf16')}")
        if page_table is None:
            self.B = int(k_cache.shape[1])
            self.max_seq = int(k_cache.shape[3])
        else:
            # paged: pools [L][n_pages][n_kv][page][d], page_table int32 [B][pages per sequence]
            self.B = int(page_table.shape[0])
            self.max_seq = int(max_seq if max_seq is not None else page_table.shape[1] * k_cache.shape[3])
        self._c = make_config(cfg, n_ctas, spin_limit_us, batch=self.B, max_seq=self.max_seq, flags=flags,
                              window=window)
        L = cfg.n_layers
        self._layers = (_abi.xlpk_layer_weights * max(L, 1))()

        def lin(name):
            gs = weights.get(name + ".gscale")   # NVFP4: the matrix scale (a one-element tensor)
            return _abi.xlpk_linear(_ptr(weights[name]), _ptr(weights.get(name + ".scale")),
                                    float(gs.reshape(-1)[0]) if gs is not None else 0.0)

        import torch

        # MoE: the C ABI takes each layer's experts as one [E][...] array per
        # projection; per-expert tensors are stacked here (kept alive until
        # create has packed them)
        stacks = []

        def stacked(prefix, n, proj):
            if n == 0:
                return _abi.xlpk_linear(0, 0)
            t = torch.stack([weights[f"{prefix}{i}.{proj}"] for i in range(n)]).contiguous()
            stacks.append(t)
            return _abi.xlpk_linear(_ptr(t), 0)

        for l in range(L):
            p = f"layers.{l}."
            lw = self._layers[l]
            lw.attn_norm_dev = _ptr(weights[p + "attn_norm"])
            lw.ffn_norm_dev = _ptr(weights[p + "ffn_norm"])
            lw.wq, lw.wk, lw.wv, lw.wo = lin(p + "wq"), lin(p + "wk"), lin(p + "wv"), lin(p + "wo")
            if getattr(cfg, "n_experts", 0):
                lw.router_dev = _ptr(weights[p + "router"])
                E, S = cfg.n_experts, cfg.n_shared_experts
                lw.we_gate = stacked(p + "experts.", E, "w_gate")
                lw.we_up = stacked(p + "experts.", E, "w_up")
                lw.we_down = stacked(p + "experts.", E, "w_down")
                lw.ws_gate = stacked(p + "shared.", S, "w_gate")
                lw.ws_up = stacked(p + "shared.", S, "w_up")
                lw.ws_down = stacked(p + "shared.", S, "w_down")
            else:
                lw.w_gate, lw.w_up, lw.w_down = lin(p + "w_gate"), lin(p + "w_up"), lin(p + "w_down")
        self._w = _abi.xlpk_weights(_ptr(weights["embed"]), _ptr(weights["final_norm"]),
                                    lin("lm_head"), self._layers)
        if page_table is None:
            self._kv = _abi.xlpk_kv(_ptr(k_cache), _ptr(v_cache), 0, 0, 0)
        else:
            self._kv = _abi.xlpk_kv(_ptr(k_cache), _ptr(v_cache), _ptr(page_table), int(k_cache.shape[3]),
                                    int(k_cache.shape[1]))
        self._refs = (weights, k_cache, v_cache, page_table)
        h = C.c_void_p()
        _check(lib.xlpk_create(C.byref(self._c), C.byref(self._w), C.byref(self._kv), C.byref(h)),
               "xlpk_create")
        self.h = h
        del stacks   # packed into the library's own buffer

    def close(self) -> None:
        if getattr(self, "h", None):
            lib.xlpk_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def info(self) -> _abi.xlpk_info:
        out = _abi.xlpk_info()
        _check(lib.xlpk_get_info(self.h, C.byref(out)), "xlpk_get_info")
        return out

    def set_state(self, tokens, seq_lens, stream=None) -> None:
        t = (C.c_int32 * self.B)(*[int(v) for v in tokens])
        s = (C.c_int32 * self.B)(*[int(v) for v in seq_lens])
        _check(lib.xlpk_set_state(self.h, t, s, _stream_handle(stream)), "xlpk_set_state")

    @staticmethod
    def _io(forced=None, logits=None, hidden=None, experts=None, trace=None, withhold_release: int = 0):
        if all(t is None for t in (forced, logits, hidden, experts, trace)) and not withhold_release:
            return None
        return _abi.xlpk_decode_io(_ptr(forced), _ptr(logits), _ptr(hidden), _ptr(experts), _ptr(trace),
                                   int(withhold_release))

    def decode(self, n_steps: int, tokens_out, forced=None, logits=None, hidden=None, experts=None,
               trace=None, stream=None, unfused: bool = False, withhold_release: int = 0) -> None:
        """xlpk_decode (or xlpk_decode_unfused); `withhold_release` is the io field
        of that name (failure-detection tests only)."""
        io = self._io(forced, logits, hidden, experts, trace, withhold_release)
        fn = lib.xlpk_decode_unfused if unfused else lib.xlpk_decode
        _check(fn(self.h, int(n_steps), _ptr(tokens_out), C.byref(io) if io is not None else None,
                  _stream_handle(stream)), "xlpk_decode_unfused" if unfused else "xlpk_decode")

    def decode_noalloc(self, n_steps: int, tokens_out, forced=None, logits=None, hidden=None,
                       stream=None) -> None:
        """xlpk_decode_noalloc: the same decode with its scratch in the library's static array."""
        io = self._io(forced, logits, hidden, None, None)
        _check(lib.xlpk_decode_noalloc(self.h, int(n_steps), _ptr(tokens_out),
                                       C.byref(io) if io is not None else None, _stream_handle(stream)),
               "xlpk_decode_noalloc")

    def debug_logits(self, logits=None, hidden=None) -> None:
        """xlpk_debug_logits: parity-mode buffers ([B][V] and [B][H] fp32 CUDA tensors,
        or None) that later decode calls overwrite with each step's values."""
        self._dbg = (logits, hidden)   # borrowed by the library until replaced
        _check(lib.xlpk_debug_logits(self.h, _ptr(logits), _ptr(hidden)), "xlpk_debug_logits")

    def verify(self, drafts, argmax_out, logits=None, hidden=None, stream=None) -> int:
        """xlpk_verify: `drafts` int32 CUDA tensor [B-1]; `argmax_out` int32 CUDA tensor [B];
        returns the number of tokens emitted (accepted drafts + the bonus token)."""
        n = C.c_int32()
        io = self._io(None, logits, hidden, None, None)
        _check(lib.xlpk_verify(self.h, _ptr(drafts), int(drafts.numel()), _ptr(argmax_out), C.byref(n),
                               C.byref(io) if io is not None else None, _stream_handle(stream)), "xlpk_verify")
        return int(n.value)

    # ---- device-resident request loop (xlpk_serve_*)

    def serve_start(self, idle_limit_us: int = 1_000_000, stream=None) -> None:
        _check(lib.xlpk_serve_start(self.h, int(idle_limit_us), _stream_handle(stream)), "xlpk_serve_start")

    def serve_post(self, n_steps: int) -> int:
        """Post n_steps more greedy steps; returns the session index of the first."""
        first = C.c_int64()
        _check(lib.xlpk_serve_post(self.h, int(n_steps), C.byref(first)), "xlpk_serve_post")
        return int(first.value)

    def serve_wait(self, first_step: int, n_steps: int, timeout_us: int = 10_000_000):
        """Wait for the posted steps; returns their tokens as a list of [B] lists."""
        out = (C.c_int32 * (int(n_steps) * self.B))()
        _check(lib.xlpk_serve_wait(self.h, int(first_step), int(n_steps), out, int(timeout_us)), "xlpk_serve_wait")
        return [[out[s * self.B + b] for b in range(self.B)] for s in range(int(n_steps))]

    def serve_stop(self) -> None:
        _check(lib.xlpk_serve_stop(self.h), "xlpk_serve_stop")

    def status(self) -> int:
        return int(lib.xlpk_get_status(self.h))

    def check(self) -> None:
        _check(lib.xlpk_get_status(self.h), "device status")

    def generate(self, tokens, seq_lens, n_steps: int, out_host, stream=None) -> None:
        """End-to-end call with host buffers; `out_host` is a pinned int32 CPU tensor [n_steps][B]."""
        t = (C.c_int32 * self.B)(*[int(v) for v in tokens])
        s = (C.c_int32 * self.B)(*[int(v) for v in seq_lens])
        _check(lib.xlpk_generate(self.h, t, s, int(n_steps),
                                 C.cast(C.c_void_p(out_host.data_ptr()), C.POINTER(C.c_int32)),
                                 _stream_handle(stream)), "xlpk_generate")
