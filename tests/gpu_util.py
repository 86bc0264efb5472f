"""Helpers for the GPU parity tests: moving seeded numpy inputs to the device
and comparing device results with the oracle's."""
import numpy as np
import torch

# Output tolerances (maximum relative error against the oracle): 1e-6 for
# fp32 outputs and 8e-3 for bf16 outputs.  The kernels are designed to match
# bit for bit, which the comparisons below also check.
TOL_F32 = 1e-6
TOL_BF16 = 8e-3


def bf16_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_host(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f32_of_bf16(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def max_rel_err(got, ref):
    got = got.astype(np.float64)
    ref = ref.astype(np.float64)
    den = np.maximum(np.abs(ref), 1e-30)
    err = np.abs(got - ref) / den
    err[(ref == 0) & (got == 0)] = 0.0
    return float(err.max()) if err.size else 0.0


def assert_f32_output(got, ref, what=""):
    got = np.asarray(got, np.float32)
    ref = np.asarray(ref, np.float32)
    assert got.shape == ref.shape
    rel = max_rel_err(got, ref)
    assert rel <= TOL_F32, "%s: max rel err %g > %g" % (what, rel, TOL_F32)
    bad = np.flatnonzero(got.view(np.uint32) != ref.view(np.uint32))
    assert bad.size == 0, "%s: %d of %d outputs differ in bits (first at %s: %r vs %r)" % (
        what, bad.size, got.size, np.unravel_index(bad[0], got.shape), got.flat[bad[0]],
        ref.flat[bad[0]])


def assert_bf16_output(got_bits, ref_bits, what=""):
    got_bits = np.asarray(got_bits, np.uint16)
    ref_bits = np.asarray(ref_bits, np.uint16)
    assert got_bits.shape == ref_bits.shape
    rel = max_rel_err(f32_of_bf16(got_bits), f32_of_bf16(ref_bits))
    assert rel <= TOL_BF16, "%s: max rel err %g > %g" % (what, rel, TOL_BF16)
    bad = np.flatnonzero(got_bits != ref_bits)
    assert bad.size == 0, "%s: %d of %d outputs differ in bits (first at %s: %#x vs %#x)" % (
        what, bad.size, got_bits.size, np.unravel_index(bad[0], got_bits.shape),
        got_bits.flat[bad[0]], ref_bits.flat[bad[0]])


def assert_exact(got, ref, what=""):
    got = np.asarray(got)
    ref = np.asarray(ref)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, "%s: %d of %d differ (first at %s: %r vs %r)" % (
        what, bad.size, got.size, np.unravel_index(bad[0], got.shape), got.flat[bad[0]],
        ref.flat[bad[0]])


# ---------------------------------------------------------------------------
# guard canaries: out-of-bounds writes show up as changed pattern bytes
# ---------------------------------------------------------------------------
GUARD_BYTES = 4096
GUARD_FILL = 0xA5


class Guard:
    """Hands out device buffers that sit between two GUARD_BYTES-long runs of
    the byte GUARD_FILL inside one allocation.  ``check()`` asserts that every
    run is unchanged, so a kernel that writes past either end of an output or
    a workspace fails the test even when the values it was asked for are
    right.  The buffer itself starts GUARD_BYTES into the allocation, so its
    alignment is the allocation's (256 bytes) whatever its size."""

    def __init__(self):
        self.bufs = []

    def empty(self, shape, dtype, fill=None):
        shape = tuple(shape) if isinstance(shape, (tuple, list)) else (shape,)
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        raw = torch.full((2 * GUARD_BYTES + n,), GUARD_FILL, dtype=torch.uint8, device="cuda")
        body = raw[GUARD_BYTES:GUARD_BYTES + n]
        if fill is not None:
            body.fill_(fill)
        self.bufs.append((raw, n, "%s %s" % (shape, dtype)))
        return body.view(dtype).view(shape)

    def copy(self, t):
        """A guarded copy of a CUDA tensor (inputs updated in place, residuals)."""
        g = self.empty(t.shape, t.dtype)
        g.copy_(t)
        return g

    def workspace(self, nbytes):
        """A guarded uint8 workspace of exactly nbytes (None when 0)."""
        return self.empty((nbytes,), torch.uint8) if nbytes else None

    def check(self):
        torch.cuda.synchronize()
        for raw, n, what in self.bufs:
            lo = raw[:GUARD_BYTES].cpu().numpy()
            hi = raw[GUARD_BYTES + n:].cpu().numpy()
            for side, run in (("before", lo), ("after", hi)):
                bad = np.flatnonzero(run != GUARD_FILL)
                assert bad.size == 0, "guard bytes %s the buffer %s were overwritten (%d bytes, " \
                    "first at offset %d)" % (side, what, bad.size, int(bad[0]))
