"""Helpers shared by the GPU parity tests: bring seeded CPU inputs to the device, compare
GPU outputs with the oracle under the stated tolerances, and guard output buffers with
canary regions."""
import numpy as np
import torch

EPS = 1e-5
RTOL, ATOL = 1e-5, 1e-6   # float outputs: |gpu - oracle| <= ATOL + RTOL |oracle|
GUARD = 256               # canary bytes on each side of guarded outputs


def bits(X_bf16_cpu):
    return X_bf16_cpu.contiguous().view(torch.int16).numpy().view(np.uint16)


def guarded_empty(shape, dtype, device="cuda", fill=0x5A):
    """A contiguous tensor of `shape` inside a larger byte buffer whose head and tail
    are filled with `fill`; check_guard() verifies they were not written."""
    n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
    raw = torch.full((GUARD + n + GUARD,), fill, dtype=torch.uint8, device=device)
    t = raw[GUARD:GUARD + n].view(dtype).view(*shape)
    t._guard_raw = raw
    t._guard_fill = fill
    return t


def check_guard(t):
    raw = t._guard_raw
    head = raw[:GUARD].cpu().numpy()
    tail = raw[-GUARD:].cpu().numpy()
    assert (head == t._guard_fill).all() and (tail == t._guard_fill).all(), "write outside the output"


def assert_float_close(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    bad = err > ATOL + RTOL * np.abs(want)
    assert not bad.any(), "%s: %d of %d outside tolerance, worst %g at %s" % (
        what, int(bad.sum()), bad.size, float(err.max()), np.unravel_index(np.argmax(err), err.shape))


def bf16_to_f32(u16):
    return (np.asarray(u16, dtype=np.uint32) << 16).view(np.float32)


def assert_bf16_match(got_u16, want_f32, want_u16, what=""):
    """bf16 outputs equal the oracle's round-to-nearest-even of its fp32 value, except
    where that fp32 value lies within 2^-21 (relative) of a bf16 rounding midpoint; there
    the two fp32 values may round to neighbouring bf16 values (1 bf16 ulp apart)."""
    got = np.asarray(got_u16, dtype=np.uint16)
    want = np.asarray(want_u16, dtype=np.uint16)
    diff = got != want
    if not diff.any():
        return
    wf = np.asarray(want_f32, dtype=np.float32)[diff].astype(np.float64)
    g = bf16_to_f32(got[diff]).astype(np.float64)
    w = bf16_to_f32(want[diff]).astype(np.float64)
    mid = (g + w) / 2
    near = np.abs(wf - mid) <= np.abs(wf) * 2.0 ** -21
    one_ulp = np.abs(got[diff].astype(np.int64) - want[diff].astype(np.int64)) == 1
    ok = near & one_ulp
    assert ok.all(), "%s: %d bf16 mismatches away from a rounding midpoint" % (what, int((~ok).sum()))
    assert diff.mean() < 1e-3, "%s: too many near-midpoint bf16 differences (%g)" % (what, diff.mean())
