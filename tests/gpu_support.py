"""Harness shared by the GPU parity tests and the smoke check.

A Harness holds one tensor collection twice: on the GPU (torch tensors,
stepped through the C ABI by the binding) and on the host (numpy arrays,
stepped by the CPU oracle).  Both sides start from the same bytes, made by
elementwise_optimizer_b200.synth, and every step both see the same gradient
bytes.  For multi-GB collections the host keeps only a deterministic index
sample of each tensor (the update is elementwise, so any element can be
stepped on its own).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import synth

TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
NPBITS = {"f32": np.uint32, "f16": np.uint16, "bf16": np.uint16}


def to_device_storage(x: np.ndarray, dtype: str, device) -> torch.Tensor:
    """float32 values (representable in dtype) -> device tensor of dtype,
    converted on the host so both sides hold identical bits."""
    st = synth.to_storage(x, dtype)
    if dtype == "bf16":
        return torch.from_numpy(st.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(st).to(device)


def storage_bits(t: torch.Tensor) -> np.ndarray:
    """Device or host tensor -> numpy array of its raw bits."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.float32:
        return t.view(torch.int32).numpy().view(np.uint32)
    return t.view(torch.int16).numpy().view(np.uint16)


def host_bits(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint32) if a.itemsize == 4 else a.view(np.uint16)


def ordered(bits: np.ndarray) -> np.ndarray:
    """Map IEEE bit patterns to integers that are monotonic in the value, so
    |ordered(a) - ordered(b)| is the distance in units in the last place."""
    width = bits.dtype.itemsize * 8
    b = bits.astype(np.int64)
    sign = np.int64(1) << (width - 1)
    return np.where(b & sign, sign - b, b + 0)


def nan_mask(bits: np.ndarray) -> np.ndarray:
    if bits.dtype == np.uint32:
        return (bits & 0x7FFFFFFF) > 0x7F800000
    return None


def ulp_distance(a_bits: np.ndarray, b_bits: np.ndarray, dtype: str) -> np.ndarray:
    """Elementwise ulp distance in the storage format (NaN vs NaN = 0,
    NaN vs number = huge)."""
    assert a_bits.dtype == b_bits.dtype
    d = np.abs(ordered(a_bits) - ordered(b_bits))
    if dtype == "f32":
        an = (a_bits & 0x7FFFFFFF) > 0x7F800000
        bn = (b_bits & 0x7FFFFFFF) > 0x7F800000
    elif dtype == "f16":
        an = (a_bits & 0x7FFF) > 0x7C00
        bn = (b_bits & 0x7FFF) > 0x7C00
    else:
        an = (a_bits & 0x7FFF) > 0x7F80
        bn = (b_bits & 0x7FFF) > 0x7F80
    d = np.where(an & bn, 0, d)
    d = np.where(an ^ bn, np.int64(1) << 40, d)
    return d


class Harness:
    """One collection on the GPU and its host mirror for the oracle.

    layout: 'separate' (one allocation per tensor, 16-byte aligned),
            'packed'   (every quantity of a dtype packed back to back in one
                        buffer: most tensors start misaligned),
            'padded'   (packed, each tensor preceded by ``pad`` elements).
    """

    def __init__(self, w: synth.Workload, device="cuda", layout="separate", pad=0,
                 sample_stride=97, sample_edge=4096, full_below=1 << 20):
        self.w = w
        self.device = torch.device(device)
        self.ademamix = w.algo == "ademamix"
        self.layout = layout
        n_t = len(w.sizes)

        # ---- device buffers ------------------------------------------------
        self.params, self.grads, self.s1, self.s2 = [], [], [], []
        self._flat = []
        if layout == "separate":
            for n, dt in zip(w.sizes, w.dtypes):
                self.params.append(torch.empty(n, dtype=TORCH[dt], device=self.device))
                self.grads.append(torch.empty(n, dtype=TORCH[dt], device=self.device))
                self.s1.append(torch.zeros(2 * n if self.ademamix else n, dtype=torch.float32,
                                           device=self.device))
                self.s2.append(torch.zeros(n, dtype=torch.float32, device=self.device))
        else:
            lead = pad if layout == "padded" else 0
            self._packed(lead)

        # ---- initial values and host mirror ------------------------------
        self.idx = []
        self.h_p, self.h_s1, self.h_s2 = [], [], []
        if not w.ring:
            init = w.params_init()
            for i in range(n_t):
                self.params[i].copy_(to_device_storage(init[i], w.dtypes[i], self.device))
                self.idx.append(None)
                self.h_p.append(synth.to_storage(init[i], w.dtypes[i]))
        else:
            self._rings = {}
            for i, (n, dt) in enumerate(zip(w.sizes, w.dtypes)):
                off = w.offset(i, 0)
                self.params[i].copy_(self._ring("param", dt)[off:off + n])
                idx = (np.arange(n, dtype=np.int64) if n <= full_below else
                       synth.sample_indices(n, sample_stride, sample_edge))
                self.idx.append(idx)
                self.h_p.append(synth.to_storage(w.ring_values("param", i, 0, idx), dt))
        for i, n in enumerate(w.sizes):
            k = n if self.idx[i] is None else len(self.idx[i])
            self.h_s1.append(np.zeros(2 * k if self.ademamix else k, np.float32))
            self.h_s2.append(np.zeros(k, np.float32))
        self._h_g = None
        self.tl = B.TensorList.from_tensors(self.params, self.grads, self.s1, self.s2)
        self.hyper = B.make_hyper(w.algo, skip_zeros=w.skip_zeros, **w.hyper)
        torch.cuda.synchronize(self.device)

    def _packed(self, lead):
        w = self.w
        for dt in sorted(set(w.dtypes)):
            members = [i for i, d in enumerate(w.dtypes) if d == dt]
            tot = sum(w.sizes[i] + lead for i in members)
            s1m = 2 if self.ademamix else 1
            bp = torch.empty(tot, dtype=TORCH[dt], device=self.device)
            bg = torch.empty(tot, dtype=TORCH[dt], device=self.device)
            b1 = torch.zeros(tot * s1m, dtype=torch.float32, device=self.device)
            b2 = torch.zeros(tot, dtype=torch.float32, device=self.device)
            self._flat += [bp, bg, b1, b2]
            pos = pos1 = 0
            views = {}
            for i in members:
                n = w.sizes[i]
                pos += lead
                pos1 += lead * s1m
                views[i] = (bp[pos:pos + n], bg[pos:pos + n],
                            b1[pos1:pos1 + s1m * n], b2[pos:pos + n])
                pos += n
                pos1 += s1m * n
            self._views = getattr(self, "_views", {})
            self._views.update(views)
        for i in range(len(w.sizes)):
            p, g, s1, s2 = self._views[i]
            self.params.append(p)
            self.grads.append(g)
            self.s1.append(s1)
            self.s2.append(s2)

    def _ring(self, which, dt):
        key = (which, dt)
        if key not in self._rings:
            pool = self.w.pool(which)
            ring = np.concatenate([pool, pool[:max(self.w.sizes)]])
            self._rings[key] = to_device_storage(
                synth.from_storage(synth.to_storage(ring, dt), dt), dt, self.device)
        return self._rings[key]

    # ---- one step on each side -------------------------------------------
    def load_grads(self, step):
        """Write step's gradients into the device buffers; keep the host copy."""
        w = self.w
        if not w.ring:
            vals = w.grads(step)
            for dt in sorted(set(w.dtypes)):
                members = [i for i, d in enumerate(w.dtypes) if d == dt]
                flat = np.concatenate([vals[i] for i in members]) if members else None
                dev = to_device_storage(flat, dt, self.device)
                pos = 0
                for i in members:
                    n = w.sizes[i]
                    self.grads[i].copy_(dev[pos:pos + n])
                    pos += n
            self._h_g = [synth.to_storage(v, d) for v, d in zip(vals, w.dtypes)]
        else:
            self._h_g = []
            for i, (n, dt) in enumerate(zip(w.sizes, w.dtypes)):
                off = w.offset(i, step)
                self.grads[i].copy_(self._ring("grad", dt)[off:off + n])
                self._h_g.append(synth.to_storage(w.ring_values("grad", i, step, self.idx[i]), dt))

    def gpu_step(self, step, plan=None, stream=None):
        if plan is not None:
            plan.step(self.hyper, step, stream)
        else:
            B.opt2s_step(self.tl, self.hyper, step, stream)

    def oracle_step(self, step):
        w = self.w
        for i, dt in enumerate(w.dtypes):
            oracle.step_f32(self.h_p[i], self._h_g[i], self.h_s1[i], self.h_s2[i], dtype=dt,
                            algo=w.algo, step=step, skip_zeros=w.skip_zeros, **w.hyper)

    def step_both(self, step, **kw):
        self.load_grads(step)
        self.gpu_step(step, **kw)
        self.oracle_step(step)

    # ---- comparison --------------------------------------------------------
    def device_sample(self, i):
        """(param bits, state1 (m[, m2]), state2) of tensor i at the host
        mirror's indices, from the device."""
        idx = self.idx[i]
        n = self.w.sizes[i]
        if idx is None:
            return storage_bits(self.params[i]), storage_bits(self.s1[i]), storage_bits(self.s2[i])
        ti = torch.from_numpy(idx).to(self.device)
        s1 = self.s1[i]
        m = s1[:n][ti]
        if self.ademamix:
            m = torch.cat([m, s1[n:][ti]])
        return storage_bits(self.params[i][ti]), storage_bits(m), storage_bits(self.s2[i][ti])

    def max_ulps(self):
        """Max ulp distance (param in its storage format, states in fp32)
        over the collection, per quantity."""
        worst = {"param": 0, "state1": 0, "state2": 0}
        for i, dt in enumerate(self.w.dtypes):
            p, s1, s2 = self.device_sample(i)
            worst["param"] = max(worst["param"], int(ulp_distance(p, host_bits(self.h_p[i]), dt).max(initial=0)))
            worst["state1"] = max(worst["state1"], int(ulp_distance(s1, host_bits(self.h_s1[i]), "f32").max(initial=0)))
            worst["state2"] = max(worst["state2"], int(ulp_distance(s2, host_bits(self.h_s2[i]), "f32").max(initial=0)))
        return worst

    def max_rel(self):
        """Max relative difference |gpu - oracle| / |oracle| of the fp32
        values of param and states (0 where both are equal, NaN = NaN)."""
        worst = 0.0
        for i, dt in enumerate(self.w.dtypes):
            p, s1, s2 = self.device_sample(i)
            pairs = [(synth.from_storage(p.view(np.float32 if dt == "f32" else np.uint16), dt),
                      synth.from_storage(self.h_p[i], dt)),
                     (s1.view(np.float32), self.h_s1[i]), (s2.view(np.float32), self.h_s2[i])]
            for a, b in pairs:
                a = a.astype(np.float64)
                b = b.astype(np.float64)
                both_nan = np.isnan(a) & np.isnan(b)
                with np.errstate(invalid="ignore", divide="ignore"):
                    r = np.where(a == b, 0.0, np.abs(a - b) / np.abs(b))
                r = np.where(both_nan, 0.0, r)
                worst = max(worst, float(np.nanmax(r, initial=0.0)) if r.size else 0.0)
                if np.any(np.isnan(a) ^ np.isnan(b)):
                    worst = float("inf")
        return worst

    def grads_unchanged(self):
        for i, dt in enumerate(self.w.dtypes):
            g = self.grads[i]
            idx = self.idx[i]
            if idx is not None:
                g = g[torch.from_numpy(idx).to(self.device)]
            if not np.array_equal(storage_bits(g), host_bits(self._h_g[i])):
                return False
        return True


class Harness8:
    """A collection for the 8-bit-state step on the GPU and its host mirror.

    Tensors of at least ``min_8bit_size`` elements keep 8-bit blockwise state
    (uint8 codes of m [| m2] and v, fp32 absmax per 2,048-element block);
    smaller ones keep fp32 state.  Everything starts at zero.  layout
    'separate' gives each buffer its own allocation; 'packed' puts every
    tensor's param/grad (per dtype), codes and fp32 state back to back in
    shared buffers, so most of them start misaligned.  Direct-mode workloads
    only (the host mirror holds every element).
    """

    def __init__(self, w: synth.Workload, device="cuda", min_8bit_size=4096, layout="separate"):
        assert not w.ring
        self.w = w
        self.device = torch.device(device)
        two = w.algo == "ademamix"
        self.bits = [8 if n >= min_8bit_size else 32 for n in w.sizes]
        self.nb = [(n + 2047) // 2048 for n in w.sizes]
        n_t = len(w.sizes)
        init = w.params_init()
        dev = self.device

        def alloc(sizes, dtype):
            """Views of one buffer (packed) or separate tensors, zero-filled."""
            if layout == "separate":
                return [torch.zeros(max(k, 0), dtype=dtype, device=dev) for k in sizes]
            buf = torch.zeros(sum(sizes) + 1, dtype=dtype, device=dev)
            out, pos = [], 1 if dtype == torch.uint8 else 0      # codes start odd
            for k in sizes:
                out.append(buf[pos:pos + k])
                pos += k
            self._keep.append(buf)
            return out

        self._keep = []
        # param / grad: packed per dtype through the 32-bit harness's helper
        self.params, self.grads = [None] * n_t, [None] * n_t
        for dt in sorted(set(w.dtypes)):
            members = [i for i, d in enumerate(w.dtypes) if d == dt]
            ps = alloc([w.sizes[i] for i in members], TORCH[dt])
            gs = alloc([w.sizes[i] for i in members], TORCH[dt])
            for k, i in enumerate(members):
                self.params[i], self.grads[i] = ps[k], gs[k]
        e8 = [i for i in range(n_t) if self.bits[i] == 8]
        e32 = [i for i in range(n_t) if self.bits[i] == 32]
        q1 = alloc([(2 if two else 1) * w.sizes[i] for i in e8], torch.uint8)
        q2 = alloc([w.sizes[i] for i in e8], torch.uint8)
        a1 = alloc([(2 if two else 1) * self.nb[i] for i in e8], torch.float32)
        a2 = alloc([self.nb[i] for i in e8], torch.float32)
        s1 = alloc([(2 if two else 1) * w.sizes[i] for i in e32], torch.float32)
        s2 = alloc([w.sizes[i] for i in e32], torch.float32)
        self.s1, self.s2, self.a1, self.a2 = [None] * n_t, [None] * n_t, [None] * n_t, [None] * n_t
        for k, i in enumerate(e8):
            self.s1[i], self.s2[i], self.a1[i], self.a2[i] = q1[k], q2[k], a1[k], a2[k]
        for k, i in enumerate(e32):
            self.s1[i], self.s2[i] = s1[k], s2[k]
        self.h_p, self.h_s1, self.h_s2, self.h_a1, self.h_a2 = [], [], [], [], []
        for i in range(n_t):
            self.params[i].copy_(to_device_storage(init[i], w.dtypes[i], dev))
            self.h_p.append(synth.to_storage(init[i], w.dtypes[i]))
            n = w.sizes[i]
            if self.bits[i] == 8:
                self.h_s1.append(np.zeros((2 if two else 1) * n, np.uint8))
                self.h_s2.append(np.zeros(n, np.uint8))
                self.h_a1.append(np.zeros((2 if two else 1) * self.nb[i], np.float32))
                self.h_a2.append(np.zeros(self.nb[i], np.float32))
            else:
                self.h_s1.append(np.zeros((2 if two else 1) * n, np.float32))
                self.h_s2.append(np.zeros(n, np.float32))
                self.h_a1.append(None)
                self.h_a2.append(None)
        self._h_g = None
        self.tl = B.TensorList8.from_tensors(self.params, self.grads, self.s1, self.s2,
                                             self.a1, self.a2)
        self.hyper = B.make_hyper(w.algo, skip_zeros=w.skip_zeros, **w.hyper)
        torch.cuda.synchronize(dev)

    def load_grads(self, step):
        vals = self.w.grads(step)
        for i, (v, dt) in enumerate(zip(vals, self.w.dtypes)):
            self.grads[i].copy_(to_device_storage(v, dt, self.device))
        self._h_g = [synth.to_storage(v, d) for v, d in zip(vals, self.w.dtypes)]

    def gpu_step(self, step, stream=None):
        B.opt2s_step_8bit(self.tl, self.hyper, step, stream)

    def oracle_step(self, step):
        w = self.w
        for i, dt in enumerate(w.dtypes):
            if self.bits[i] == 8:
                oracle.step_8bit(self.h_p[i], self._h_g[i], self.h_s1[i], self.h_s2[i],
                                 self.h_a1[i], self.h_a2[i], dtype=dt, algo=w.algo, step=step,
                                 skip_zeros=w.skip_zeros, **w.hyper)
            else:
                oracle.step_f32(self.h_p[i], self._h_g[i], self.h_s1[i], self.h_s2[i], dtype=dt,
                                algo=w.algo, step=step, skip_zeros=w.skip_zeros, **w.hyper)

    def step_both(self, step):
        self.load_grads(step)
        self.gpu_step(step)
        self.oracle_step(step)

    def mismatches(self):
        """(tensor, quantity, count of differing elements) for every array
        that differs from the host mirror bit for bit."""
        torch.cuda.synchronize(self.device)
        bad = []
        for i in range(len(self.w.sizes)):
            pairs = [("param", storage_bits(self.params[i]), host_bits(self.h_p[i]))]
            if self.bits[i] == 8:
                pairs += [("codes1", self.s1[i].cpu().numpy(), self.h_s1[i]),
                          ("codes2", self.s2[i].cpu().numpy(), self.h_s2[i]),
                          ("absmax1", storage_bits(self.a1[i]), host_bits(self.h_a1[i])),
                          ("absmax2", storage_bits(self.a2[i]), host_bits(self.h_a2[i]))]
            else:
                pairs += [("state1", storage_bits(self.s1[i]), host_bits(self.h_s1[i])),
                          ("state2", storage_bits(self.s2[i]), host_bits(self.h_s2[i]))]
            for name, a, b in pairs:
                if not np.array_equal(a, b):
                    bad.append((i, name, int(np.count_nonzero(a != b))))
        return bad

    def grads_unchanged(self):
        return all(np.array_equal(storage_bits(g), host_bits(h)) for g, h in zip(self.grads, self._h_g))
