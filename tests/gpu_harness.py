"""Shared helpers of the GPU parity tests: run the library through its C ABI on
seeded synthetic inputs and compare every stage with the CPU oracle."""
from __future__ import annotations

import ctypes
import math
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import long_context_attention_rkv_b200 as rkv
import oracle
import synth

# tolerances of the parity contract
IDX_TIE_BAND = 1e-4         # relative gap between the k-th and (k+1)-th oracle distance
CODE_LSB_FRACTION = 1e-3    # codes may differ by one step on at most this fraction of elements
RECON_ABS = 1e-2            # reconstructed K/V
ATTN_ABS = 2e-3             # decode output (fp32 output; bf16 output adds half a bf16 ulp)


def to_dev(arr: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(arr)
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(a).cuda()


def config(wl: synth.Workload, lengths, max_len=None, out_dtype=rkv.RKV_DTYPE_F32, flags=0, batch=None,
           ref_bits=0, coder=0):
    return rkv.make_config(head_dim=wl.head_dim, n_kv_heads=wl.n_kv_heads, n_q_heads=wl.n_q_heads, k=wl.k,
                           bits=wl.bits, stride0=wl.stride0, batch=len(lengths) if batch is None else batch,
                           max_len=max(max(lengths), 1) if max_len is None else max_len,
                           refs_per_phase=wl.refs_per_phase, in_dtype=wl.dtype_code, out_dtype=out_dtype,
                           flags=flags, ref_bits=ref_bits, coder=coder)


class DeviceRun:
    """One layer compressed on the GPU through the C ABI."""

    def __init__(self, wl: synth.Workload, K: np.ndarray, V: np.ndarray, lengths, out_dtype=rkv.RKV_DTYPE_F32,
                 flags=0, start_lengths=None, ref_bits=0, coder=None):
        """lengths: the bound (capacity) lengths; start_lengths: a shorter prefix to compress
        first (grown later with append_until); ref_bits 4: the int4 reference store; coder:
        (oracle.Coder K, oracle.Coder V) for the learned-coder shapes."""
        self.wl = wl
        self.lengths = list(lengths)
        self.coder = coder
        self.cfg = config(wl, lengths, max_len=K.shape[2], out_dtype=out_dtype, flags=flags, ref_bits=ref_bits,
                          coder=0 if coder is None else 1)
        self.layer = rkv.Layer(self.cfg, self.lengths)
        if coder is not None:
            ws = [w for c in coder for w in (c.Wg, c.Wu, c.Wo, c.Wd)]
            self.layer.set_coder([to_dev(oracle.bf16_round(w)) for w in ws])
        self.Kd = to_dev(K)
        self.Vd = to_dev(V)
        self.cur = list(self.lengths if start_lengths is None else start_lengths)
        if start_lengths is not None:
            self.layer.set_lengths(self.cur)
        self.layer.build_refs(self.Kd, self.Vd)
        self.layer.compress(self.Kd, self.Vd)
        torch.cuda.synchronize()
        err = self.layer.device_error()
        assert err == 0, f"device error {rkv.STATUS.get(err, err)}"

    def append_until(self, target):
        """Appends each sequence's next tokens (from the same K, V) until it reaches target."""
        B, Hkv = len(self.lengths), self.wl.n_kv_heads
        bi = torch.arange(B, device="cuda").repeat_interleave(Hkv)
        hi = torch.arange(Hkv, device="cuda").repeat(B)
        while any(c < t for c, t in zip(self.cur, target)):
            act = [1 if self.cur[b] < target[b] else 0 for b in range(B)]
            pos = torch.tensor([min(self.cur[b], self.Kd.shape[2] - 1) for b in range(B)],
                               device="cuda").repeat_interleave(Hkv)
            Kn = self.Kd[bi, hi, pos].contiguous()
            Vn = self.Vd[bi, hi, pos].contiguous()
            self.layer.append(Kn, Vn, act)
            self.cur = [c + a for c, a in zip(self.cur, act)]
        torch.cuda.synchronize()
        err = self.layer.device_error()
        assert err == 0, f"device error {rkv.STATUS.get(err, err)}"

    def _read(self, ptr, nbytes, dtype, shape):
        if nbytes == 0:
            return np.zeros(shape, dtype=dtype)
        off = ptr - self.layer.cache.data_ptr()
        assert 0 <= off and off + nbytes <= self.layer.cache.numel()
        raw = self.layer.cache[off:off + nbytes].cpu().numpy()
        return raw.view(dtype).reshape(shape)

    def unit(self, b: int, h: int) -> dict:
        v = self.layer.unit(b, h)
        D, R, C, k = self.wl.head_dim, v.n_ref, v.n_cmp, v.k
        refs = {}
        if v.ref_bits == 4:
            # the int4 reference store: codes and scales as stored, and their stored values
            for side, cp, sp in (("K", v.ref_K, v.ref_scale_K), ("V", v.ref_V, v.ref_scale_V)):
                codes = self._read(cp, R * D // 2, np.uint8, (R, D // 2))
                scales = self._read(sp, 2 * R * (D // 32), np.uint16, (R, D // 32))
                refs["ref_codes" + side] = codes
                refs["ref_scales" + side] = scales
                refs["ref" + side] = oracle.dequantize_rows(codes, scales, D, 4, 32) if R else \
                    np.zeros((0, D), np.float32)
        else:
            refs["refK"] = self._read(v.ref_K, 2 * R * D, np.uint16, (R, D))
            refs["refV"] = self._read(v.ref_V, 2 * R * D, np.uint16, (R, D))
        return dict(
            n=v.n, R=R, C=C, ref_bits=v.ref_bits, **refs,
            hn=self._read(v.ref_half_norm, 4 * R, np.float32, (R,)),
            pos=self._read(v.ref_pos, 4 * R, np.int32, (R,)),
            codesK=self._read(v.codes_K, C * v.code_bytes, np.uint8, (C, v.code_bytes)),
            codesV=self._read(v.codes_V, C * v.code_bytes, np.uint8, (C, v.code_bytes)),
            scalesK=self._read(v.scale_K, 2 * C * v.n_groups, np.uint16, (C, v.n_groups)),
            scalesV=self._read(v.scale_V, 2 * C * v.n_groups, np.uint16, (C, v.n_groups)),
            idx=self._read(v.idx, 2 * C * k, np.uint16, (C, k)),
        )

    def decode(self, q: np.ndarray) -> np.ndarray:
        qd = to_dev(q)
        dt = torch.float32 if self.cfg.out_dtype == rkv.RKV_DTYPE_F32 else torch.bfloat16
        out = torch.empty((len(self.lengths), self.wl.n_q_heads, self.wl.head_dim), dtype=dt, device="cuda")
        self.layer.decode(qd, out)
        torch.cuda.synchronize()
        err = self.layer.device_error()
        assert err == 0, f"device error {rkv.STATUS.get(err, err)}"
        return out.float().cpu().numpy()

    def reconstruct(self, b: int, h: int, positions=None):
        n = self.lengths[b]
        npos = n if positions is None else len(positions)
        K = torch.empty((max(npos, 1), self.wl.head_dim), dtype=torch.float32, device="cuda")
        V = torch.empty_like(K)
        pd = None if positions is None else to_dev(np.asarray(positions, dtype=np.int32))
        self.layer.reconstruct(b, h, pd, npos, K, V, rkv.RKV_DTYPE_F32)
        torch.cuda.synchronize()
        assert self.layer.device_error() == 0
        return K[:npos].cpu().numpy(), V[:npos].cpu().numpy()


# --- oracle-side comparisons --------------------------------------------------------------

def unit_rows(wl: synth.Workload, K: np.ndarray, V: np.ndarray, b: int, h: int, n: int):
    """Float rows (exact input values) of one unit."""
    return synth.as_f32(wl, K[b, h, :n]), synth.as_f32(wl, V[b, h, :n])


def slots_of(positions: np.ndarray, ref_pos: np.ndarray) -> np.ndarray:
    return positions - np.searchsorted(ref_pos, positions, side="right")


def _unpack(codes: np.ndarray, D: int, bits: int) -> np.ndarray:
    if bits == 8:
        return codes.view(np.int8).astype(np.int64)
    lo = (codes & 0xF).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    out = np.empty(codes.shape[:-1] + (D,), dtype=np.int64)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out)


def stored_values(refs: np.ndarray) -> np.ndarray:
    """Reference values as fp32: bf16 bits widened, or already values (int4 store)."""
    return refs if refs.dtype == np.float32 else oracle.bf16_value(refs)


def check_refs(wl, g: dict, Xk, Xv):
    ref_pos = oracle.schedule(len(Xk), wl.stride0, wl.refs_per_phase)
    assert np.array_equal(g["pos"], ref_pos)
    if g["ref_bits"] == 4:
        for side, X in (("K", Xk), ("V", Xv)):
            codes, scales, vals, ov = oracle.build_refs_quantized(X, ref_pos)
            assert ov == 0
            assert np.array_equal(g["ref_codes" + side], codes), f"reference {side} codes differ"
            assert np.array_equal(g["ref_scales" + side], scales), f"reference {side} scales differ"
            assert np.array_equal(g["ref" + side], vals)
    else:
        assert np.array_equal(g["refK"], oracle.build_refs(Xk, ref_pos))
        assert np.array_equal(g["refV"], oracle.build_refs(Xv, ref_pos))
    rv = stored_values(g["refK"]).astype(np.float64)
    np.testing.assert_allclose(g["hn"], 0.5 * (rv * rv).sum(axis=1), rtol=2e-6, atol=1e-30)
    return ref_pos


def check_compress(wl, g: dict, Xk, Xv, positions=None, stats=None, coder=None):
    """Selection (tie-band aware) and codes of compressed positions against the oracle."""
    n = len(Xk)
    ref_pos = oracle.schedule(n, wl.stride0, wl.refs_per_phase)
    cpos, _ = oracle.positions_split(n, ref_pos)
    if positions is None:
        positions = cpos
    positions = np.asarray(positions, dtype=np.int32)
    if len(positions) == 0:
        return
    slots = slots_of(positions, ref_pos)
    refK = g["refK"]
    refV = g["refV"]
    gidx = g["idx"][slots]
    oidx, okeff, odist = oracle.select(Xk[positions], positions, refK, ref_pos, wl.k)
    k = wl.k
    mism = 0
    for t in np.nonzero(np.any(gidx != oidx, axis=1))[0]:
        mism += 1
        ke = okeff[t]
        dk, dk1 = odist[t, ke - 1], odist[t, ke]
        assert ke < k + 1 and not math.isnan(dk1), f"selection differs at position {positions[t]} with no tie"
        assert dk1 - dk <= IDX_TIE_BAND * dk, (
            f"selection differs outside the tie band at position {positions[t]}: "
            f"gpu {gidx[t]} oracle {oidx[t]} d_k={dk} d_k+1={dk1}")
        sel = gidx[t][gidx[t] != oracle.SENTINEL]
        assert len(sel) == ke and np.all(np.diff(sel.astype(int)) > 0) and np.all(ref_pos[sel] < positions[t])
        rv = stored_values(refK)
        worst = max(oracle.l2(Xk[positions[t]], rv[j]) for j in sel)
        assert worst <= dk1 * (1 + IDX_TIE_BAND)
    # codes: the oracle's encoder fed the GPU's index sets
    if coder is not None:
        ek = oracle.encode_latent(Xk[positions], refK, gidx, wl.bits, coder[0], wl.group)
        ev = oracle.encode_latent(Xv[positions], refV, gidx, wl.bits, coder[1], wl.group)
    else:
        ek = oracle.encode(Xk[positions], refK, gidx, wl.bits, wl.group)
        ev = oracle.encode(Xv[positions], refV, gidx, wl.bits, wl.group)
    assert ek["overflow"] == 0 and ev["overflow"] == 0
    D = wl.head_dim
    # learned-coder shapes and the identity coder share one contract: scales bit-exact, codes
    # equal except for one step on at most CODE_LSB_FRACTION of the elements (the latent's
    # power-of-two scales leave its codes a reproducible function of z)
    for name, e in (("K", ek), ("V", ev)):
        assert np.array_equal(g["scales" + name][slots], e["scales"]), f"{name} scales differ"
        gc = _unpack(g["codes" + name][slots], D, wl.bits)
        oc = _unpack(e["codes"], D, wl.bits)
        diff = np.abs(gc - oc)
        assert diff.max(initial=0) <= 1, f"{name} codes differ by more than one step"
        assert diff.astype(bool).mean() <= CODE_LSB_FRACTION
    if stats is not None:
        stats["tokens"] = stats.get("tokens", 0) + len(positions)
        stats["idx_tie_mismatch"] = stats.get("idx_tie_mismatch", 0) + mism


def oracle_decode_on_gpu_cache(wl, g: dict, q_group: np.ndarray, coder=None):
    """The oracle's reconstruction and attention over the cache the GPU produced."""
    n = g["n"]
    if n == 0:
        return np.zeros((q_group.shape[0], wl.head_dim))
    Kh, Vh = oracle.unit_cache_rows(n, g["pos"], g["refK"], g["refV"], g["idx"], g["codesK"], g["scalesK"],
                                    g["codesV"], g["scalesV"], wl.bits, wl.group, coder=coder)
    return oracle.attention(q_group.astype(np.float64), Kh, Vh)


def check_decode(run: DeviceRun, q: np.ndarray, units=None, threads=8):
    """Decode output of every (or the listed) unit against the oracle on the GPU's cache."""
    wl = run.wl
    out = run.decode(q)
    qf = synth.as_f32(wl, q)
    G = wl.n_q_heads // wl.n_kv_heads
    units = [(b, h) for b in range(len(run.lengths)) for h in range(wl.n_kv_heads)] if units is None else units
    gus = {u: run.unit(*u) for u in units}

    def one(u):
        b, h = u
        return u, oracle_decode_on_gpu_cache(wl, gus[u], qf[b, h * G:(h + 1) * G], run.coder)

    with ThreadPoolExecutor(threads) as ex:
        refs = dict(ex.map(one, units))
    worst = 0.0
    for (b, h), ref in refs.items():
        got = out[b, h * G:(h + 1) * G].astype(np.float64)
        if run.cfg.out_dtype == rkv.RKV_DTYPE_F32:
            tol = ATTN_ABS
        else:
            tol = ATTN_ABS + np.abs(ref) * 2.0 ** -8          # half an ulp of bf16 on top
        err = np.abs(got - ref)
        assert np.all(err <= tol), f"decode unit {(b, h)}: max err {err.max()}"
        worst = max(worst, float(err.max(initial=0)))
    return worst


def check_reconstruct(run: DeviceRun, g: dict, b: int, h: int, positions=None):
    wl = run.wl
    n = g["n"]
    Kh, Vh = oracle.unit_cache_rows(n, g["pos"], g["refK"], g["refV"], g["idx"], g["codesK"], g["scalesK"],
                                    g["codesV"], g["scalesV"], wl.bits, wl.group, coder=run.coder)
    Kg, Vg = run.reconstruct(b, h, positions)
    sel = np.arange(n) if positions is None else np.asarray(positions)
    np.testing.assert_allclose(Kg, Kh[sel], atol=RECON_ABS, rtol=0)
    np.testing.assert_allclose(Vg, Vh[sel], atol=RECON_ABS, rtol=0)
    return float(max(np.abs(Kg - Kh[sel]).max(initial=0), np.abs(Vg - Vh[sel]).max(initial=0)))


def sample_positions(wl, n: int, n_uniform=2048, seed=0):
    """Deterministic row sample: the first k*s positions, phase boundaries +-2, uniform rows."""
    ref_pos = oracle.schedule(n, wl.stride0, wl.refs_per_phase)
    cpos, is_ref = oracle.positions_split(n, ref_pos)
    pick = set(range(min(n, wl.k * wl.stride0)))
    if wl.refs_per_phase:
        for j in range(0, len(ref_pos), wl.refs_per_phase):
            for d in (-2, -1, 1, 2):
                pick.add(int(ref_pos[j]) + d)
    rng = np.random.default_rng(seed)
    if len(cpos):
        pick.update(int(p) for p in rng.choice(cpos, min(n_uniform, len(cpos)), replace=False))
    pick.add(n - 1)
    return np.array(sorted(p for p in pick if 0 <= p < n and not is_ref[p]), dtype=np.int32)
