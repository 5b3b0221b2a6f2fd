"""Helpers shared by the GPU tests: moving raw host codes to torch device
tensors, running one decode step (reshape_and_cache of the new token, then
decode) through the library, and the oracle's side of the same step."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_448_b200 as pk
from paged_kv_cache_448_b200 import workloads as wl

# Element-wise acceptance: |gpu - ref| <= ATOL + RTOL * |ref| (the stated
# max-abs and relative bounds read element-wise: the output's own rounding to
# bf16 alone reaches 3.9e-3 at |ref| in [1, 2)), and, tighter, within one ulp
# or ATOL of the oracle's result rounded to the output type.
TOL = {"f16": (2e-3, 1e-2), "bf16": (2e-3, 1e-2), "e4m3": (3e-2, 3e-2)}

_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16}


def dev(codes: np.ndarray, dt: str, device="cuda") -> torch.Tensor:
    """Raw host codes -> device tensor of the storage dtype (E4M3 as uint8)."""
    a = np.ascontiguousarray(codes)
    if dt == "e4m3":
        return torch.from_numpy(a.view(np.uint8)).to(device)
    return torch.from_numpy(a.view(np.int16)).view(_TORCH[dt]).to(device)


def host_codes(t: torch.Tensor) -> np.ndarray:
    """Device tensor -> raw host codes (uint16 for 16-bit types, uint8 for E4M3)."""
    t = t.detach().contiguous().cpu()
    if t.dtype in (torch.float16, torch.bfloat16):
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.view(torch.uint8).numpy()


def i32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def f32(a, device="cuda"):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def within_tol(gpu: np.ndarray, ref: np.ndarray, cache_dtype: str):
    atol, rtol = TOL[cache_dtype]
    err = np.abs(gpu - ref)
    ok = err <= atol + rtol * np.abs(ref)
    return bool(ok.all()), float(err.max(initial=0.0))


def _out_dtype(gpu: np.ndarray, cache_dtype: str) -> str:
    """The 16-bit type the output was stored in: the cache's for a 16-bit
    cache; for E4M3 (bf16 or f16 query) bf16 if every value is a bf16 value."""
    if cache_dtype in ("f16", "bf16"):
        return cache_dtype
    t = torch.from_numpy(np.ascontiguousarray(gpu))
    return "bf16" if torch.equal(t.to(torch.bfloat16).double(), t) else "f16"


def rounding_check(gpu: np.ndarray, ref: np.ndarray, cache_dtype: str, out_dtype=None):
    """The tighter check: the GPU's 16-bit output against the oracle's result
    correctly rounded (nearest even) to that type. Each element must be within
    one unit in the last place of the rounded value, or within the absolute
    bound (2e-3 for 16-bit caches, 3e-2 for E4M3). Returns the elements
    that fail (an index array) and the largest distance in ulps."""
    od = out_dtype or _out_dtype(gpu, cache_dtype)
    codes = oracle.round_to(ref, od)
    r = oracle.decode_array(codes, od)
    # one ulp at r: the distance to the next code of larger magnitude
    nxt = oracle.decode_array((codes & 0x7FFF) + 1, od)
    ulp = np.abs(nxt - np.abs(r))
    d = np.abs(gpu - r)
    bound = np.maximum(ulp, TOL[cache_dtype][0])
    return np.argwhere(d > bound), float((d / ulp).max(initial=0.0))


def assert_close(gpu: np.ndarray, ref: np.ndarray, cache_dtype: str, what="", out_dtype=None):
    """|gpu - ref| <= atol + rtol |ref| element-wise (ref: the oracle's fp64
    result), and the rounding check above against the oracle's rounded
    output."""
    ok, worst = within_tol(gpu, ref, cache_dtype)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    if not ok:
        atol, rtol = TOL[cache_dtype]
        bad = np.argwhere(np.abs(gpu - ref) > atol + rtol * np.abs(ref))
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} elements out of tolerance; first {i}: "
                             f"gpu={gpu[i]!r} ref={ref[i]!r} (max abs err {worst:.3g})")
    bad, ulps = rounding_check(gpu, ref, cache_dtype, out_dtype)
    if len(bad):
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} elements more than 1 ulp and "
                             f"{TOL[cache_dtype][0]} from the rounded oracle result; first {i}: "
                             f"gpu={gpu[i]!r} ref={ref[i]!r} (max {ulps:.3g} ulp)")


GUARD = 4096            # bytes of sentinel before and after a guarded buffer
SENTINEL = 0xA7


class Guarded:
    """A device buffer with GUARD sentinel bytes on either side, standing in
    for an out-of-bounds checker: any stray write of a kernel just before or
    after the buffer changes a sentinel. `t` is the buffer itself (aligned to
    256 bytes within the allocation)."""

    def __init__(self, shape, dtype, device="cuda", fill=None):
        esz = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) * esz
        self.raw = torch.full((GUARD + n + GUARD,), SENTINEL, dtype=torch.uint8, device=device)
        self.n = n
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def check(self, what=""):
        head = self.raw[:GUARD]
        tail = self.raw[GUARD + self.n:]
        assert bool((head == SENTINEL).all()) and bool((tail == SENTINEL).all()), \
            f"{what}: a write landed outside the buffer (guard bytes changed)"


def guarded_workspace(nbytes, device="cuda"):
    """A workspace of nbytes inside guard bytes, error word zeroed."""
    g = Guarded((max(nbytes, 256),), torch.uint8, device=device)
    g.t.fill_(0xFF)              # everything past the header starts as garbage
    g.t[:256].zero_()
    return g


class GpuStep:
    """Device copies of a workload and the library calls of one decode step."""

    def __init__(self, sp: wl.Spec, st: wl.Structure, hd: wl.HostData, device="cuda"):
        self.sp, self.st, self.hd = sp, st, hd
        self.q = dev(hd.query, sp.q_dtype, device)
        self.kc = dev(hd.key_cache, sp.cache_dtype, device)
        self.vc = dev(hd.value_cache, sp.cache_dtype, device)
        self.nk = dev(hd.new_key, sp.q_dtype, device)
        self.nv = dev(hd.new_value, sp.q_dtype, device)
        self.ks, self.vs = f32(hd.k_scale, device), f32(hd.v_scale, device)
        self.bt = i32(st.block_tables, device)
        self.cl = i32(sp.context_lens, device)
        slots = pk.build_slot_mapping(st.block_tables, st.positions, sp.block_size)
        self.slots = i32(slots, device)
        self.out_g = Guarded(tuple(self.q.shape), self.q.dtype, device)
        self.out = self.out_g.t
        self.max_ctx = int(sp.context_lens.max())

    def reshape(self):
        pk.reshape_and_cache(self.nk, self.nv, self.kc, self.vc, self.slots, k_scale=self.ks,
                             v_scale=self.vs)

    def decode(self, partition_tokens=None, workspace=None):
        """One decode; afterwards the workspace's error word must be clear (a
        table error or a pipeline wait that gave up raises PagedError)."""
        sp = self.sp
        p = sp.partition_tokens if partition_tokens is None else partition_tokens
        wsg = None
        if workspace is None:
            wsg = guarded_workspace(pk.decode_workspace_size(
                sp.num_seqs, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size,
                self.max_ctx, p, pk.dtype_code(self.kc)))
            workspace = wsg.t
        out = pk.decode(self.out, self.q, self.kc, self.vc, self.bt, self.cl, self.max_ctx,
                        sp.scale, k_scale=self.ks, v_scale=self.vs, partition_tokens=p,
                        workspace=workspace)
        pk.decode_check(workspace)
        self.out_g.check("decode output")
        if wsg is not None:
            wsg.check("decode workspace")
        return out

    def out_f64(self) -> np.ndarray:
        return self.out.double().cpu().numpy()


def oracle_step(sp: wl.Spec, st: wl.Structure, hd: wl.HostData, seqs=None):
    """The oracle's reshape_and_cache of the new tokens followed by decode.
    Returns (key_cache, value_cache, out[S, H, D] fp64) on the host."""
    kc, vc = hd.key_cache.copy(), hd.value_cache.copy()
    slots = oracle.slot_mapping(st.block_tables, st.positions, sp.block_size)
    oracle.reshape_and_cache(hd.new_key, hd.new_value, kc, vc, slots, block_size=sp.block_size,
                             kv_dtype=sp.q_dtype, cache_dtype=sp.cache_dtype,
                             k_scale=hd.k_scale, v_scale=hd.v_scale)
    sel = slice(None) if seqs is None else np.asarray(seqs)
    out = oracle.decode(hd.query[sel], kc, vc, st.block_tables[sel], sp.context_lens[sel],
                        scale=np.float32(sp.scale), q_dtype=sp.q_dtype,
                        cache_dtype=sp.cache_dtype, k_scale=hd.k_scale, v_scale=hd.v_scale)
    return kc, vc, out
