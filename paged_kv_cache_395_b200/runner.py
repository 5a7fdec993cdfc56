"""Replay a workload (``workloads.Workload``) on the GPU through the C ABI.

Uploads every operation's arrays once, owns the device KV pool, and runs
setup / step operations with ``pa_reshape_and_cache``, ``pa_block_copy`` and
``pa_decode`` -- or, for a step whose append ends with its sequences' new
tokens, those tokens and the decode with one ``pa_decode_append`` call.
Optionally converts the pool to int8 (``pa_quantize_int8``) after setup.
"""
from __future__ import annotations

import numpy as np
import torch

from . import pa
from . import workloads as W

NAN_BITS = {torch.float16: 0x7E00, torch.bfloat16: 0x7FC0}


def torch_dtype(name: str) -> torch.dtype:
    return {"float32": torch.float32, "float16": torch.float16, "bfloat16": torch.bfloat16}[name]


def to_device(a: np.ndarray, dtype_name: str | None, device) -> torch.Tensor:
    if dtype_name == "bfloat16" and a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


class DeviceWorkload:
    def __init__(self, w: W.Workload, device="cuda", fill_nan: bool = True, steps=None):
        self.w = w
        self.device = torch.device(device)
        self.dtype = torch_dtype(w.dtype)
        shape = (w.num_blocks, w.num_kv_heads, w.block_size, w.head_dim)
        self.kc = torch.empty(shape, dtype=self.dtype, device=self.device)
        self.vc = torch.empty_like(self.kc)
        self.fill(fill_nan)
        self.k_scales = self.v_scales = None
        self.kc8 = self.vc8 = None
        self.setup = [self._upload(op) for op in w.setup]
        idx = range(len(w.steps)) if steps is None else steps
        self.steps = {i: [self._upload(op) for op in w.steps[i]] for i in idx}
        # steps whose append ends with one new token per decoded sequence, at its last
        # position (pa_decode_append can take those tokens)
        self.new_tokens = {i: new_token_split(w.steps[i]) for i in idx}
        self.out = {}

    def fill(self, nan: bool):
        if nan and self.dtype in NAN_BITS:
            self.kc.view(torch.int16).fill_(NAN_BITS[self.dtype])
            self.vc.view(torch.int16).fill_(NAN_BITS[self.dtype])
        else:
            self.kc.fill_(float("nan") if nan else 0.0)
            self.vc.fill_(float("nan") if nan else 0.0)

    def _upload(self, op):
        d, n = self.device, self.w.dtype
        if isinstance(op, W.Reshape):
            return ("reshape", to_device(op.k, n, d), to_device(op.v, n, d),
                    torch.from_numpy(op.slot_mapping).to(d))
        if isinstance(op, W.Copy):
            return ("copy", torch.from_numpy(np.ascontiguousarray(op.pairs)).to(d))
        q = to_device(op.q, n, d)
        return ("decode", q, torch.from_numpy(op.block_tables).to(d),
                torch.from_numpy(op.seq_lens).to(d), int(op.max_seq_len), torch.empty_like(q))

    def quantize_int8(self):
        """Replace the pool by its int8 form (one scale per (block, KV head))."""
        N, H = self.kc.shape[:2]
        self.kc8 = torch.empty(self.kc.shape, dtype=torch.int8, device=self.device)
        self.vc8 = torch.empty_like(self.kc8)
        self.k_scales = torch.empty((N, H), dtype=torch.float32, device=self.device)
        self.v_scales = torch.empty_like(self.k_scales)
        pa.pa_quantize_int8(self.kc, self.kc8, self.k_scales)
        pa.pa_quantize_int8(self.vc, self.vc8, self.v_scales)

    def quantize_int4(self):
        """Replace the pool by its 4-bit form (two values per byte, one scale per
        (block, KV head)); the caches become uint8 [N][H_kv][16][d/2]."""
        N, H, bs, d = self.kc.shape
        self.kc8 = torch.empty((N, H, bs, d // 2), dtype=torch.uint8, device=self.device)
        self.vc8 = torch.empty_like(self.kc8)
        self.k_scales = torch.empty((N, H), dtype=torch.float32, device=self.device)
        self.v_scales = torch.empty_like(self.k_scales)
        pa.pa_quantize_int4(self.kc, self.kc8, self.k_scales)
        pa.pa_quantize_int4(self.vc, self.vc8, self.v_scales)

    def workspace_for(self, op, partition_size, int8=False, algo=pa.PA_ALGO_AUTO):
        """int8: the quantised pool (int8, or 4-bit after quantize_int4) is decoded."""
        _, q, bt, _, mx, _ = op
        kc = self.kc8 if int8 else self.kc
        n = pa.pa_decode_workspace_size(q, kc, bt, mx, partition_size,
                                        self.k_scales if int8 else None,
                                        self.v_scales if int8 else None, algo)
        return pa.alloc_workspace(n, self.device)

    def run(self, op, partition_size=0, workspace=None, int8=False, algo=pa.PA_ALGO_AUTO,
            stream=None, out_f32=False):
        """out_f32: decode into a new float32 tensor (the fp32 result before the
        output's rounding) instead of the step's own output."""
        kind = op[0]
        if kind == "reshape":
            _, k, v, s = op
            pa.pa_reshape_and_cache(k, v, self.kc, self.vc, s, stream=stream)
        elif kind == "copy":
            if op[1].numel():
                pa.pa_block_copy(self.kc, self.vc, op[1], stream=stream)
        else:
            _, q, bt, sl, mx, out = op
            if out_f32:
                out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
            if workspace is None and partition_size != 0:
                workspace = self.workspace_for(op, partition_size, int8, algo)
            kc, vc = (self.kc8, self.vc8) if int8 else (self.kc, self.vc)
            pa.pa_decode(out, q, kc, vc, bt, sl, self.w.scale, mx,
                         self.k_scales if int8 else None, self.v_scales if int8 else None,
                         partition_size, workspace, algo, stream=stream)
            return out

    def run_setup(self):
        for op in self.setup:
            self.run(op)

    def run_step(self, i, partition_size=0, int8=False, algo=pa.PA_ALGO_AUTO, decode=True,
                 out_f32=False, fused=False):
        """fused: a step whose append ends with its sequences' new tokens runs the
        rest of the append (if any) with pa_reshape_and_cache, then those tokens and
        the decode with one pa_decode_append call."""
        if fused and decode and not int8 and self.new_tokens.get(i) is not None:
            for op in self.steps[i][:-2]:
                self.run(op)
            (_, k, v, s), dec = self.steps[i][-2:]
            _, q, bt, sl, mx, out = dec
            T, B = k.shape[0], q.shape[0]
            if T > B:
                pa.pa_reshape_and_cache(k[:T - B], v[:T - B], self.kc, self.vc, s[:T - B])
            if out_f32:
                out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
            ws = self.workspace_for(dec, partition_size, False, algo) if partition_size != 0 else None
            pa.pa_decode_append(out, q, k[T - B:], v[T - B:], s[T - B:], self.kc, self.vc, bt, sl, self.w.scale,
                                mx, partition_size, ws, algo)
            return out
        out = None
        for op in self.steps[i]:
            if op[0] == "decode":
                if decode:
                    out = self.run(op, partition_size, None, int8, algo, out_f32=out_f32)
            else:
                self.run(op)
        return out

    def decode_again(self, i, partition_size=0, int8=False, algo=pa.PA_ALGO_AUTO, out_f32=False):
        """Repeat step i's decode alone (its appends already ran)."""
        op = [o for o in self.steps[i] if o[0] == "decode"][0]
        return self.run(op, partition_size, None, int8, algo, out_f32=out_f32)


def new_token_split(ops):
    """For a step [..., Reshape, Decode] of single-token decode whose Reshape ends
    with one token per sequence at its last position (slot of position
    seq_lens[b] - 1 under the block table; no token for an empty sequence), the
    number of leading tokens before them; else None."""
    if len(ops) < 2 or not isinstance(ops[-2], W.Reshape) or not isinstance(ops[-1], W.Decode):
        return None
    r, d = ops[-2:]
    if d.q.ndim != 3:
        return None
    B, T = d.q.shape[0], len(r.slot_mapping)
    if T < B:
        return None
    slots = r.slot_mapping[T - B:]
    L = d.seq_lens.astype(np.int64)
    for b in range(B):
        if L[b] <= 0:
            if slots[b] >= 0:
                return None
            continue
        pos = L[b] - 1
        if slots[b] != int(d.block_tables[b, pos // W.BLOCK_SIZE]) * W.BLOCK_SIZE + pos % W.BLOCK_SIZE:
            return None
    return T - B


class StepCalls:
    """Pre-marshalled C-ABI calls for every step, so a timed loop costs one
    ctypes call per library entry point and nothing else on the host."""

    def __init__(self, dw: DeviceWorkload, partition_size=-1, int8=False, algo=pa.PA_ALGO_AUTO,
                 stream=None, flags=0, append_flags=0, fused=False, prompt_flags=0):
        """flags: pa_decode flags; append_flags: pa_reshape_and_cache_ex flags
        (PA_APPEND_OVERLAP_PREVIOUS only for recipes whose appends never touch
        what the previous step's decode reads, ``appends_overlap_previous``).
        fused: steps whose append ends with their sequences' new tokens issue the
        leading tokens (prompts of admitted sequences) with pa_reshape_and_cache_ex
        and prompt_flags, then one pa_decode_append call for the new tokens and the
        decode (its launches as pa_decode_append_fused reports)."""
        import ctypes
        self.dw = dw
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        sp = ctypes.c_void_p(self.stream.cuda_stream)
        w = dw.w
        kc, vc = (dw.kc8, dw.vc8) if int8 else (dw.kc, dw.vc)
        ks = dw.k_scales if int8 else None
        vs = dw.v_scales if int8 else None
        ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
        if (append_flags or prompt_flags) and not getattr(w, "appends_overlap_previous", False):
            raise ValueError("this recipe's appends may touch what the previous decode reads")
        aflags = int(append_flags)
        self.fused_steps = 0
        # one workspace, sized for the largest step
        need = 0
        for ops in dw.steps.values():
            for op in ops:
                if op[0] == "decode":
                    _, q, bt, _, mx, _ = op
                    need = max(need, pa.pa_decode_workspace_size(q, kc, bt, mx, partition_size,
                                                                 ks, vs, algo))
        self.workspace = pa.alloc_workspace(need, dw.device)
        self.keep = []
        self.calls = {}
        self.launches = {}
        for i, ops in dw.steps.items():
            calls, launches = [], 0
            lead = dw.new_tokens.get(i) if fused and not int8 else None
            if lead is not None:
                N, H, bs, d = dw.kc.shape
                for op in ops[:-2]:  # copy-on-write copies before the append
                    if op[0] != "copy":
                        raise ValueError("a fused step takes only block copies before its append")
                    n = op[1].numel() // 2
                    if n:
                        args = (ptr(dw.kc), ptr(dw.vc), None, None, ptr(op[1]), n, H, d, bs, N,
                                pa.dtype_code(dw.kc.dtype), sp)
                        calls.append(("copy", pa.lib.pa_block_copy, args))
                        launches += 1
                (_, k, v, s), (_, q, bt, sl, mx, out) = ops[-2:]
                if lead:
                    args = (ptr(k), ptr(v), ptr(dw.kc), ptr(dw.vc), ptr(s), lead, H, d, bs, N,
                            pa.dtype_code(k.dtype), k.stride(0), v.stride(0), int(prompt_flags), sp)
                    calls.append(("reshape", pa.lib.pa_reshape_and_cache_ex, args))
                    launches += 1
                kn, vn, sn = k[lead:], v[lead:], s[lead:]
                p = pa.make_params(q, kc, bt, mx, None, None, partition_size, self.workspace, algo, flags)
                self.keep.append(p)
                dl = pa.lib.pa_decode_launches(ctypes.byref(p), ptr(q))
                if dl < 0:
                    raise pa.PaError(dl, "pa_decode_launches")
                one = pa.lib.pa_decode_append_fused(ctypes.byref(p), ptr(q), ptr(kn), ptr(vn), kn.stride(0),
                                                    vn.stride(0))
                if one < 0:
                    raise pa.PaError(one, "pa_decode_append_fused")
                args = (ptr(out), ptr(q), ptr(kn), ptr(vn), ptr(sn), kn.stride(0), vn.stride(0), ptr(kc),
                        ptr(vc), ptr(bt), ptr(sl), ctypes.c_float(w.scale), ctypes.byref(p), sp)
                calls.append(("decode", pa.lib.pa_decode_append, args))
                # the append kernel unless fused, then the decode's own launches
                launches += (0 if one == 1 else 1) + dl
                self.fused_steps += one == 1
                self.calls[i] = calls
                self.launches[i] = launches
                continue
            for op in ops:
                if op[0] == "reshape":
                    _, k, v, s = op
                    N, H, bs, d = dw.kc.shape
                    args = (ptr(k), ptr(v), ptr(dw.kc), ptr(dw.vc), ptr(s), k.shape[0], H, d, bs, N,
                            pa.dtype_code(k.dtype), k.stride(0), v.stride(0), aflags, sp)
                    calls.append(("reshape", pa.lib.pa_reshape_and_cache_ex, args))
                    launches += 1 if k.shape[0] else 0
                elif op[0] == "copy":
                    n = op[1].numel() // 2
                    if n:
                        N, H, bs, d = dw.kc.shape
                        args = (ptr(dw.kc), ptr(dw.vc), None, None, ptr(op[1]), n, H, d, bs, N,
                                pa.dtype_code(dw.kc.dtype), sp)
                        calls.append(("copy", pa.lib.pa_block_copy, args))
                        launches += 1
                else:
                    _, q, bt, sl, mx, out = op
                    p = pa.make_params(q, kc, bt, mx, ks, vs, partition_size, self.workspace, algo,
                                       flags)
                    self.keep.append(p)
                    dl = pa.lib.pa_decode_launches(ctypes.byref(p), ptr(q))
                    if dl < 0:
                        raise pa.PaError(dl, "pa_decode_launches")
                    args = (ptr(out), ptr(q), ptr(kc), ptr(vc), ptr(bt), ptr(sl),
                            ctypes.c_float(w.scale), ctypes.byref(p), sp)
                    calls.append(("decode", pa.lib.pa_decode, args))
                    launches += dl
            self.calls[i] = calls
            self.launches[i] = launches

    def run_decode_only(self, i):
        """Issue only the decode call of step i (kernel timing)."""
        for name, fn, args in self.calls[i]:
            if name == "decode":
                rc = fn(*args)
                if rc != 0:
                    raise pa.PaError(rc, name)

    def run(self, i, on_decode=None):
        """Issue step i; ``on_decode(before: bool)`` brackets the decode call."""
        for name, fn, args in self.calls[i]:
            if name == "decode" and on_decode is not None:
                on_decode(True)
            rc = fn(*args)
            if rc != 0:
                raise pa.PaError(rc, name)
            if name == "decode" and on_decode is not None:
                on_decode(False)
