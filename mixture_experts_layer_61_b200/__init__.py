"""Python binding of libmoe.so -- the B200 (sm_100a) MoE layer forward.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors; the work is enqueued on the current
torch stream.  There is no CPU fallback: without the built library, or on a
device other than sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")
_lib = None

BF16, FP32 = 0, 1
SOFTMAX, SIGMOID = 0, 1
STATUS = {0: "MOE_OK", -1: "MOE_ERR_ARG", -2: "MOE_ERR_WORKSPACE", -3: "MOE_ERR_CUDA",
          -4: "MOE_ERR_TIMEOUT", -5: "MOE_ERR_DEVICE"}


class MoeError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)} ({_lib.moe_status_string(code).decode()})")


class MoeConfig(ctypes.Structure):
    """moe_config_t (include/moe.h)."""
    _fields_ = [(n, ctypes.c_int) for n in
                ("T", "H", "E", "K", "I", "n_shared", "I_shared", "tile_B", "score_fn", "renorm", "dtype",
                 "pad_mode")]

    def __repr__(self):
        return "MoeConfig(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


BLOCKWISE, MAXVALUE = 0, 1  # padding schemes of the alignment


def config(T, H, E, K, I, n_shared=0, I_shared=0, tile_B=16, score_fn=SOFTMAX, renorm=1, dtype=BF16,
           pad_mode=BLOCKWISE):
    if isinstance(dtype, torch.dtype):
        dtype = BF16 if dtype == torch.bfloat16 else FP32
    return MoeConfig(T, H, E, K, I, n_shared, I_shared, tile_B, score_fn, renorm, dtype, pad_mode)


def lib():
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with "
                              "`python -m mixture_experts_layer_61_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        C = ctypes.POINTER(MoeConfig)
        sig = {
            "moe_status_string": (ctypes.c_char_p, [I]),
            "moe_padded_rows_max": (ctypes.c_int64, [C]),
            "moe_workspace_size": (S, [C]),
            "moe_gemm_workspace_size": (S, []),
            "moe_router_gemm": (I, [C, P, P, P, P, S, P]),
            "moe_route": (I, [C, P, P, P, P]),
            "moe_route_k": (I, [C, P, P, P, P, P]),
            "moe_align_pad": (I, [C, P, P, P, P, P, P, P, P]),
            "moe_permute": (I, [C, P, P, P, P, P]),
            "moe_grouped_ffn": (I, [C, P, P, P, P, P, P, P, S, P]),
            "moe_grouped_gate_up": (I, [C, P, P, P, P, P, S, P]),
            "moe_grouped_down": (I, [C, P, P, P, P, P, S, P]),
            "moe_combine": (I, [C, P, P, P, P, P, P]),
            "moe_layer_forward": (I, [C, P, P, P, P, P, P, P, P, P, S, P, P]),
            "moe_layer_forward_k": (I, [C, P, P, P, P, P, P, P, P, P, P, S, P, P]),
            "moe_quantize_fp8": (I, [ctypes.c_int64, I, I, P, P, P, P]),
            "moe_grouped_ffn_fp8": (I, [C, P, P, P, P, P, P, P, P, P, P, S, P]),
            "dense_ffn_fp8": (I, [I, I, I, P, P, P, P, P, P, P, S, P]),
            "dense_ffn_fp8_workspace_size": (S, [I, I, I]),
            "moe_permute_e4m3x2": (I, [C, P, P, P, P, P, P]),
            "moe_layer_forward_fp8": (I, [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P, P]),
            "dense_ffn_workspace_size": (S, [I, I, I, I]),
            "dense_ffn": (I, [I, I, I, I, P, P, P, P, P, S, P]),
            "moe_check_status": (I, [P, P]),
            "moe_set_wait_limit_ns": (None, [ctypes.c_uint64]),
            "moe_debug_withhold_first_load": (None, [I]),
            "moe_set_token_tile_cap": (I, [I]),
            "moe_set_programmatic_launch": (None, [I]),
            "moe_set_split_tail": (I, [I]),
            "moe_set_cta_pairs": (None, [I]),
            "moe_set_shared_sms": (I, [I]),
            "moe_shared_sms": (I, [C]),
            "moe_ffn_fused": (I, [C]),
            "moe_layer_logits_offset": (ctypes.c_int64, [C]),
            "moe_kernel_launch_count": (ctypes.c_uint64, []),
            "moe_tp_shard": (I, [I, I, I, I, I, I, P, P, P, P, P]),
            "moe_layer_forward_partial": (I, [C, P, P, P, P, P, P, P, P, P, P, S, P, P]),
            "moe_tp_reduce": (I, [I, ctypes.POINTER(ctypes.c_void_p), ctypes.c_longlong, I, P, P]),
            "moe_layer_forward_partial_front": (I, [C, P, P, P, P, P, P, P, P, S, P, P]),
            "moe_layer_forward_partial_down": (I, [C, P, I, I, P, P, S, P]),
            "moe_tp_gather": (I, [I, ctypes.POINTER(ctypes.c_void_p), I, I, I, P, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_functions():
    """Names of the functions include/moe.h declares."""
    with open(HEADER) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_\w+|dense_ffn\w*)\s*\(", text)))


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(rc, what):
    if rc != 0:
        raise MoeError(rc, what)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def _act_dtype(cfg):
    return torch.bfloat16 if cfg.dtype == BF16 else torch.float32


# ------------------------------------------------------------ workspaces

def workspace_size(cfg):
    n = lib().moe_workspace_size(ctypes.byref(cfg))
    if n == 0:
        raise MoeError(-1, "moe_workspace_size")
    return n


def gemm_workspace_size():
    return lib().moe_gemm_workspace_size()


def dense_workspace_size(T, H, I, dtype=BF16):
    return lib().dense_ffn_workspace_size(T, H, I, dtype)


def alloc_workspace(nbytes, device="cuda"):
    """A zeroed workspace (the library keeps its control words zero after each call)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def padded_rows_max(cfg):
    return int(lib().moe_padded_rows_max(ctypes.byref(cfg)))


# ------------------------------------------------------------- the steps

def router_gemm(cfg, x, w_r, ws, logits=None):
    _need_cuda(x, w_r, ws)
    if logits is None:
        logits = torch.empty((cfg.T, cfg.E), dtype=torch.float32, device=x.device)
    _check(lib().moe_router_gemm(ctypes.byref(cfg), _p(x), _p(w_r), _p(logits), _p(ws), ws.numel(), _stream()),
           "moe_router_gemm")
    return logits


def route(cfg, logits, ids=None, w=None, k=None):
    """Top-K ids and gate weights; k (device int32 [T], optional) gives each
    token its own expert count (per-token dynamic K, empty slots -1)."""
    _need_cuda(logits, k)
    if ids is None:
        ids = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device=logits.device)
        w = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device=logits.device)
    _check(lib().moe_route_k(ctypes.byref(cfg), _p(logits), _p(k), _p(ids), _p(w), _stream()), "moe_route_k")
    return ids, w


def align_buffers(cfg, device):
    """Output buffers of align_pad for this configuration."""
    Pm = padded_rows_max(cfg)
    nblk = (Pm + cfg.tile_B - 1) // cfg.tile_B
    return dict(counts=torch.empty(cfg.E, dtype=torch.int32, device=device),
                offsets=torch.empty(cfg.E + 1, dtype=torch.int32, device=device),
                sorted_ids=torch.empty(max(Pm, 1), dtype=torch.int32, device=device),
                block_expert=torch.empty(max(nblk, 1), dtype=torch.int32, device=device),
                pos=torch.empty(max(cfg.T * cfg.K, 1), dtype=torch.int32, device=device),
                scalars=torch.zeros(4, dtype=torch.int32, device=device))


def align_pad(cfg, ids, out=None):
    _need_cuda(ids)
    Pm = padded_rows_max(cfg)
    nblk = (Pm + cfg.tile_B - 1) // cfg.tile_B
    if out is None:
        out = align_buffers(cfg, ids.device)
    out = dict(out)
    _check(lib().moe_align_pad(ctypes.byref(cfg), _p(ids), _p(out["counts"]), _p(out["offsets"]),
                               _p(out["sorted_ids"]), _p(out["block_expert"]), _p(out["pos"]),
                               _p(out["scalars"]), _stream()), "moe_align_pad")
    out["sorted_ids"] = out["sorted_ids"][:Pm]
    out["block_expert"] = out["block_expert"][:nblk]
    out["pos"] = out["pos"][:cfg.T * cfg.K]
    return out


def permute(cfg, x, sorted_ids, scalars, x_perm=None):
    _need_cuda(x, sorted_ids, scalars)
    if x_perm is None:
        x_perm = torch.empty((max(padded_rows_max(cfg), 1), cfg.H), dtype=x.dtype, device=x.device)
    _check(lib().moe_permute(ctypes.byref(cfg), _p(x), _p(sorted_ids), _p(scalars), _p(x_perm), _stream()),
           "moe_permute")
    return x_perm


def grouped_ffn(cfg, x_perm, w13, w2, offsets, ws, act=None, y_perm=None):
    _need_cuda(x_perm, w13, w2, offsets, ws)
    Pm = max(padded_rows_max(cfg), 1)
    if act is None:
        act = torch.empty((Pm, cfg.I), dtype=x_perm.dtype, device=x_perm.device)
    if y_perm is None:
        y_perm = torch.empty((Pm, cfg.H), dtype=x_perm.dtype, device=x_perm.device)
    _check(lib().moe_grouped_ffn(ctypes.byref(cfg), _p(x_perm), _p(w13), _p(w2), _p(offsets), _p(act), _p(y_perm),
                                 _p(ws), ws.numel(), _stream()), "moe_grouped_ffn")
    return y_perm, act


def grouped_gate_up(cfg, x_perm, w13, offsets, ws, act):
    _need_cuda(x_perm, w13, offsets, ws, act)
    _check(lib().moe_grouped_gate_up(ctypes.byref(cfg), _p(x_perm), _p(w13), _p(offsets), _p(act), _p(ws),
                                     ws.numel(), _stream()), "moe_grouped_gate_up")
    return act


def grouped_down(cfg, act, w2, offsets, ws, y_perm):
    _need_cuda(act, w2, offsets, ws, y_perm)
    _check(lib().moe_grouped_down(ctypes.byref(cfg), _p(act), _p(w2), _p(offsets), _p(y_perm), _p(ws),
                                  ws.numel(), _stream()), "moe_grouped_down")
    return y_perm


def combine(cfg, y_perm, pos, w, shared_out=None, out=None):
    _need_cuda(y_perm, pos, w, shared_out)
    if out is None:
        out = torch.empty((cfg.T, cfg.H), dtype=y_perm.dtype, device=y_perm.device)
    _check(lib().moe_combine(ctypes.byref(cfg), _p(y_perm), _p(pos), _p(w), _p(shared_out), _p(out), _stream()),
           "moe_combine")
    return out


def layer_forward(cfg, x, w_r, w13, w2, ws, w13_sh=None, w2_sh=None, logits_override=None, out=None,
                  stats=None, k=None):
    """The whole layer; k (device int32 [T], optional): per-token dynamic K."""
    _need_cuda(x, w_r, w13, w2, ws, w13_sh, w2_sh, logits_override, stats, k)
    if out is None:
        out = torch.empty((cfg.T, cfg.H), dtype=x.dtype, device=x.device)
    _check(lib().moe_layer_forward_k(ctypes.byref(cfg), _p(x), _p(w_r), _p(w13), _p(w2), _p(w13_sh), _p(w2_sh),
                                     _p(logits_override), _p(k), _p(out), _p(ws), ws.numel(), _p(stats),
                                     _stream()),
           "moe_layer_forward_k")
    return out


def quantize_fp8(w):
    """Row-wise FP8 E4M3 codes and fp32 scales of a weight tensor whose last
    dimension is the input features (rows = everything else), on the device:
    returns (codes uint8 of w's shape, scales float32 of w.shape[:-1])."""
    _need_cuda(w)
    cols = w.shape[-1]
    rows = w.numel() // cols
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    sc = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    dt = BF16 if w.dtype == torch.bfloat16 else FP32
    _check(lib().moe_quantize_fp8(rows, cols, dt, _p(w), _p(q), _p(sc), _stream()), "moe_quantize_fp8")
    return q, sc


def dense_ffn_fp8(x, q13, s13, q2, s2, ws, out=None):
    _need_cuda(x, q13, s13, q2, s2, ws)
    T, H = x.shape
    I = q2.shape[1]
    if out is None:
        out = torch.empty((T, H), dtype=x.dtype, device=x.device)
    _check(lib().dense_ffn_fp8(T, H, I, _p(x), _p(q13), _p(s13), _p(q2), _p(s2), _p(out), _p(ws), ws.numel(),
                               _stream()), "dense_ffn_fp8")
    return out


def dense_fp8_workspace_size(T, H, I):
    return int(lib().dense_ffn_fp8_workspace_size(T, H, I))


def permute_e4m3x2(cfg, x, sorted_ids, scalars, x_codes=None, x_scales=None):
    """moe_permute for the FP8-weight path: the permuted rows split exactly
    into E4M3 hi codes (rows [0, P_max)), lo codes (rows [P_max, 2 P_max))
    and power-of-two row scales."""
    _need_cuda(x, sorted_ids, scalars)
    Pm = max(padded_rows_max(cfg), 1)
    if x_codes is None:
        x_codes = torch.empty((2 * Pm, cfg.H), dtype=torch.uint8, device=x.device)
    if x_scales is None:
        x_scales = torch.empty((Pm,), dtype=torch.float32, device=x.device)
    _check(lib().moe_permute_e4m3x2(ctypes.byref(cfg), _p(x), _p(sorted_ids), _p(scalars), _p(x_codes),
                                    _p(x_scales), _stream()), "moe_permute_e4m3x2")
    return x_codes, x_scales


def grouped_ffn_fp8(cfg, x_codes, x_scales, q13, s13, q2, s2, offsets, ws, act, y_perm):
    _need_cuda(x_codes, x_scales, q13, s13, q2, s2, offsets, ws, act, y_perm)
    _check(lib().moe_grouped_ffn_fp8(ctypes.byref(cfg), _p(x_codes), _p(x_scales), _p(q13), _p(s13), _p(q2),
                                     _p(s2), _p(offsets), _p(act), _p(y_perm), _p(ws), ws.numel(), _stream()),
           "moe_grouped_ffn_fp8")
    return y_perm, act


def layer_forward_fp8(cfg, x, w_r, q13, s13, q2, s2, ws, q13_sh=None, s13_sh=None, q2_sh=None, s2_sh=None,
                      logits_override=None, out=None, stats=None, k=None):
    """The layer with FP8 expert weights (codes and row scales from quantize_fp8)."""
    _need_cuda(x, w_r, q13, s13, q2, s2, ws, q13_sh, s13_sh, q2_sh, s2_sh, logits_override, stats, k)
    if out is None:
        out = torch.empty((cfg.T, cfg.H), dtype=x.dtype, device=x.device)
    _check(lib().moe_layer_forward_fp8(ctypes.byref(cfg), _p(x), _p(w_r), _p(q13), _p(s13), _p(q2), _p(s2),
                                       _p(q13_sh), _p(s13_sh), _p(q2_sh), _p(s2_sh), _p(logits_override), _p(k),
                                       _p(out), _p(ws), ws.numel(), _p(stats), _stream()),
           "moe_layer_forward_fp8")
    return out


def dense_ffn(x, w13, w2, ws, out=None):
    _need_cuda(x, w13, w2, ws)
    T, H = x.shape
    I = w2.shape[1]
    dt = BF16 if x.dtype == torch.bfloat16 else FP32
    if out is None:
        out = torch.empty((T, H), dtype=x.dtype, device=x.device)
    _check(lib().dense_ffn(T, H, I, dt, _p(x), _p(w13), _p(w2), _p(out), _p(ws), ws.numel(), _stream()),
           "dense_ffn")
    return out


def check_status(ws):
    """Synchronise the current stream; raise MoeError if a device wait timed out."""
    _check(lib().moe_check_status(_p(ws), _stream()), "moe_check_status")


def set_wait_limit_ns(ns):
    lib().moe_set_wait_limit_ns(int(ns))


def set_token_tile_cap(n):
    """Force the grouped GEMM's token-tile cap (32/64/128/256; 0 = automatic)."""
    _check(lib().moe_set_token_tile_cap(int(n)), "moe_set_token_tile_cap")


def set_split_tail(mode=1):
    """GEMM tail schedule: 1 aligned k-slices of the last partial wave (the
    library default), 0 contiguous stream-K over the last one to two waves."""
    _check(lib().moe_set_split_tail(int(mode)), "moe_set_split_tail")


def set_programmatic_launch(enable=True):
    """Programmatic dependent launch between the layer's kernels (default on)."""
    lib().moe_set_programmatic_launch(1 if enable else 0)


def layer_logits(cfg, ws):
    """View of the fp32 router logits [T,E] of the last layer_forward in `ws`."""
    off = int(lib().moe_layer_logits_offset(ctypes.byref(cfg)))
    if off < 0:
        raise MoeError(-1, "moe_layer_logits_offset")
    n = cfg.T * cfg.E * 4
    return ws[off:off + n].view(torch.float32).view(cfg.T, cfg.E)


def ffn_fused(cfg):
    """True when the layer's expert FFN runs as one fused (decode) launch."""
    return bool(lib().moe_ffn_fused(ctypes.byref(cfg)))


def set_cta_pairs(enable=True):
    """2-SM (CTA pair) GEMM tiles for bf16 at the 256-token cap (default on)."""
    lib().moe_set_cta_pairs(1 if enable else 0)


def set_shared_sms(n=0):
    """SMs for the shared experts running beside the routed ones: 0 = cost
    model (default), n > 0 = fixed share, -1 = run them after, serially."""
    _check(lib().moe_set_shared_sms(int(n)), "moe_set_shared_sms")


def shared_sms(cfg):
    """SMs the shared experts of `cfg` get (0 = serial or none)."""
    return int(lib().moe_shared_sms(ctypes.byref(cfg)))


def debug_withhold_first_load(enable=True):
    lib().moe_debug_withhold_first_load(1 if enable else 0)


def kernel_launch_count():
    return int(lib().moe_kernel_launch_count())


class MoELayer:
    """Owns a configuration and its workspace; forward() runs the whole layer."""

    def __init__(self, cfg, weights, device="cuda"):
        self.cfg = cfg
        self.w = weights
        self.ws = alloc_workspace(workspace_size(cfg), device)
        self.stats = torch.zeros(4, dtype=torch.int32, device=device)

    def forward(self, x, logits_override=None, out=None):
        return layer_forward(self.cfg, x, self.w["w_r"], self.w["w13"], self.w["w2"], self.ws,
                             self.w.get("w13_sh"), self.w.get("w2_sh"), logits_override, out, self.stats)


# ------------------------------------------------ tensor parallelism over I
# Rank r of n holds, for every routed expert and for the shared FFN, the gate
# rows [r*I/n, (r+1)*I/n) of W1, the same rows of W3 and the same columns of
# W2 (talk notes, "Demystifying the Mixture of Experts Serving Tax",
# "Balls-Bins-Buckets framework": the n_tp GPUs are the buckets under TP); the
# router is whole on every rank.  Each rank computes an fp32 partial output,
# one all-reduce sums them ("Key findings" 3), and one rounding follows.

def tp_config(cfg, n_ranks):
    """The per-rank configuration of `cfg` split over I into n_ranks."""
    I_sh = cfg.n_shared * cfg.I_shared
    if n_ranks < 1 or cfg.I % n_ranks or I_sh % n_ranks:
        raise ValueError("I and the shared FFN's width must split evenly over the ranks")
    return MoeConfig(cfg.T, cfg.H, cfg.E, cfg.K, cfg.I // n_ranks, 1 if I_sh else 0, I_sh // n_ranks,
                     cfg.tile_B, cfg.score_fn, cfg.renorm, cfg.dtype, cfg.pad_mode)


def tp_shard(w13, w2, rank, n_ranks):
    """Rank `rank`'s slice of w13 [E,2I,H] / w2 [E,H,I] (or one dense FFN
    [2I,H] / [H,I]): new device tensors [E,2I/n,H] / [E,H,I/n]."""
    _need_cuda(w13, w2)
    dense = w13.dim() == 2
    E = 1 if dense else w13.shape[0]
    H, I = w2.shape[-2], w2.shape[-1]
    n = I // n_ranks if n_ranks > 0 else 0
    lead = () if dense else (E,)
    a = torch.empty(lead + (2 * n, H), dtype=w13.dtype, device=w13.device)
    b = torch.empty(lead + (H, n), dtype=w2.dtype, device=w2.device)
    dt = BF16 if w13.dtype == torch.bfloat16 else FP32
    _check(lib().moe_tp_shard(E, H, I, dt, rank, n_ranks, _p(w13), _p(w2), _p(a), _p(b), _stream()),
           "moe_tp_shard")
    return a, b


def layer_forward_partial(cfg, x, w_r, w13, w2, ws, w13_sh=None, w2_sh=None, logits_override=None, out=None,
                          stats=None, k=None):
    """This rank's fp32 partial output [T,H] for its slice (cfg from tp_config)."""
    _need_cuda(x, w_r, w13, w2, ws, w13_sh, w2_sh, logits_override, out, stats, k)
    if out is None:
        out = torch.empty((cfg.T, cfg.H), dtype=torch.float32, device=x.device)
    _check(lib().moe_layer_forward_partial(ctypes.byref(cfg), _p(x), _p(w_r), _p(w13), _p(w2), _p(w13_sh),
                                           _p(w2_sh), _p(logits_override), _p(k), _p(out), _p(ws), ws.numel(),
                                           _p(stats), _stream()),
           "moe_layer_forward_partial")
    return out


def tp_reduce(parts, out=None, dtype=torch.bfloat16):
    """out = sum of the fp32 partial outputs in list order, rounded once to
    dtype (the parts may be other GPUs' memory mapped here)."""
    _need_cuda(out, *parts)
    count = parts[0].numel()
    if any(p_.numel() != count or p_.dtype != torch.float32 for p_ in parts):
        raise ValueError("parts must be fp32 tensors of one size")
    if out is None:
        out = torch.empty(parts[0].shape, dtype=dtype, device=parts[0].device)
    ptrs = (ctypes.c_void_p * len(parts))(*[p_.data_ptr() for p_ in parts])
    dt = BF16 if out.dtype == torch.bfloat16 else FP32
    _check(lib().moe_tp_reduce(len(parts), ptrs, count, dt, _p(out), _stream()), "moe_tp_reduce")
    return out


def tp_allreduce(partial, group=None):
    """Sums the ranks' fp32 partial outputs in place across `group` (the
    collective step of TP over I; NCCL on GPUs)."""
    import torch.distributed as dist

    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


def layer_forward_partial_front(cfg, x, w_r, w13, ws, w13_sh=None, w2_sh=None, logits_override=None, stats=None,
                                k=None):
    """This rank's layer up to the routed gate/up and the shared FFN (results
    in `ws`), for the down projection by output-feature blocks."""
    _need_cuda(x, w_r, w13, ws, w13_sh, w2_sh, logits_override, stats, k)
    _check(lib().moe_layer_forward_partial_front(ctypes.byref(cfg), _p(x), _p(w_r), _p(w13), _p(w13_sh), _p(w2_sh),
                                                 _p(logits_override), _p(k), _p(ws), ws.numel(), _p(stats),
                                                 _stream()),
           "moe_layer_forward_partial_front")


def layer_forward_partial_down(cfg, w2, chunk, n_chunks, ws, part=None):
    """Down projection + combine of output features block `chunk` of
    n_chunks into part [T, H/n_chunks] fp32 (unrounded)."""
    _need_cuda(w2, ws, part)
    if part is None:
        part = torch.empty((cfg.T, cfg.H // n_chunks), dtype=torch.float32, device=w2.device)
    _check(lib().moe_layer_forward_partial_down(ctypes.byref(cfg), _p(w2), int(chunk), int(n_chunks), _p(part),
                                                _p(ws), ws.numel(), _stream()), "moe_layer_forward_partial_down")
    return part


def tp_gather(parts, out):
    """out [T, H] = the column blocks `parts` ([T, H/n] fp32 each) side by side,
    rounded once to out's dtype."""
    _need_cuda(out, *parts)
    T, H = out.shape
    ptrs = (ctypes.c_void_p * len(parts))(*[p_.data_ptr() for p_ in parts])
    dt = BF16 if out.dtype == torch.bfloat16 else FP32
    _check(lib().moe_tp_gather(len(parts), ptrs, T, H, dt, _p(out), _stream()), "moe_tp_gather")
    return out


def tp_allreduce_async(partial, group=None):
    """Starts the sum of `partial` across `group` (in place) and returns the
    pending work, or None when there is nothing to sum (one rank)."""
    import torch.distributed as dist

    if dist.is_initialized() and dist.get_world_size(group) > 1:
        return dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group, async_op=True)
    return None


def tp_overlapped_allreduce(parts, produce, group=None):
    """The overlap protocol of TP over I: for each output-feature block c in
    order, produce(c) enqueues the block's partial into parts[c], then its
    all-reduce starts (asynchronously, beside the next block's work); all of
    them are waited for before returning."""
    works = []
    for c in range(len(parts)):
        produce(c)
        works.append(tp_allreduce_async(parts[c], group))
    for w_ in works:
        if w_ is not None:
            w_.wait()
    return parts


def tp_layer_forward_overlapped(cfg_local, x, w_r, w13, w2, ws, w13_sh=None, w2_sh=None, n_chunks=4,
                                logits_override=None, parts=None, out=None, group=None, k=None):
    """One layer under TP over I with the all-reduce overlapped with the down
    projection: the front part, then per block of H/n_chunks output features
    the down projection + combine into its fp32 part and that part's
    all-reduce, then the concatenation and rounding.  At decode sizes (the
    fused expert FFN) it is tp_layer_forward."""
    if ffn_fused(cfg_local):
        return tp_layer_forward(cfg_local, x, w_r, w13, w2, ws, w13_sh, w2_sh, logits_override, out=out,
                                group=group, k=k)
    if parts is None:
        parts = [torch.empty((cfg_local.T, cfg_local.H // n_chunks), dtype=torch.float32, device=x.device)
                 for _ in range(n_chunks)]
    if out is None:
        out = torch.empty((cfg_local.T, cfg_local.H), dtype=x.dtype, device=x.device)
    layer_forward_partial_front(cfg_local, x, w_r, w13, ws, w13_sh, w2_sh, logits_override, k=k)
    tp_overlapped_allreduce(parts, lambda c: layer_forward_partial_down(cfg_local, w2, c, len(parts), ws, parts[c]),
                            group)
    return tp_gather(parts, out)


def tp_layer_forward(cfg_local, x, w_r, w13, w2, ws, w13_sh=None, w2_sh=None, logits_override=None,
                     partial=None, out=None, group=None, k=None):
    """One layer under TP over I on this rank: partial output (kernels), the
    all-reduce over `group`, then the rounding (kernel)."""
    partial = layer_forward_partial(cfg_local, x, w_r, w13, w2, ws, w13_sh, w2_sh, logits_override, partial,
                                    k=k)
    tp_allreduce(partial, group)
    return tp_reduce([partial], out, dtype=x.dtype)
