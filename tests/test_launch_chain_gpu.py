"""Small problems chain their kernels as programmatic dependents: the scan
starts while the builder finishes, and the readout while the scan runs (its
queries, keys and values load, and its items without an inter phase run,
before it waits for the prefixes).  Results must not depend on what ran
before on the stream or on how the calls were issued.

Each case is computed once on its own (fresh buffers, the device idle), then
(a) again, back to back with another input on the same stream, into the same
output, state and workspace buffers, and (b) from a CUDA graph replayed on
new inputs.  Two MMA-issuing threads add into one tensor-memory accumulator
in an order that depends on timing, so repeated calls agree up to the
rounding order of fp32 sums, not bit for bit: every result must equal the
first within that (a few units in the last place), far below what a read of
stale or unfinished data (another input's state, a prefix before the scan
wrote it) would give.  Parity of the same calls with the oracle:
test_parity_gpu.py, test_from_state_gpu.py and test_mg_gpu.py.
"""
from __future__ import annotations

import pytest

from kernelized_linear_attention_fwd_b200 import inputs

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():  # collected on CPU machines, run only with a GPU
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

import kernelized_linear_attention_fwd_b200 as K  # noqa: E402
from kernelized_linear_attention_fwd_b200.csrc import build as kbuild  # noqa: E402


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()
    K.load_library()
    yield
    assert K.kata_get_device_status() == 0


# (kind, B, H, T, d): every one small enough for the chained launches (the
# builder's and the readout's work items at most one per SM)
CASES = [
    ("forward", 2, 4, 4096, 32),   # the small d = 32 workload's shape
    ("forward", 1, 2, 2048, 64),
    ("forward", 1, 3, 700, 16),    # one ragged segment: the scan runs for the export
    ("mg2", 1, 2, 1500, 64),       # two factors, ragged last segment
    ("from_state", 1, 2, 1500, 64),
]


class Case:
    """Static buffers of one case and the call that fills them."""

    def __init__(self, kind, B, H, T, d):
        self.kind = kind
        dev = torch.device("cuda")
        self.q, self.k, self.v = (torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev)
                                  for _ in range(3))
        self.out = torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev)
        self.S = torch.empty((B, H, d * d, d), dtype=torch.float32, device=dev)
        self.Z = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
        if kind == "mg2":
            nbytes = K.kata_mg_chunked_forward_workspace_bytes(B, H, T, d, d, 64, 2, 1)
        else:
            nbytes = K.kata_chunked_forward_workspace_bytes(B, H, T, d, d, 64, 1)
        self.ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=dev)
        if kind == "from_state":  # the state of a 900-token history, a fixed input
            hq, hk, hv = inputs.make_qkv_device(B, H, 900, d, d, seed=91)
            self.S_in, self.Z_in = K.kata_chunked_state(hk, hv, C=64)

    def load(self, x):
        for dst, src in zip((self.q, self.k, self.v), x):
            dst.copy_(src)

    def call(self):
        if self.kind == "forward":
            K.kata_chunked_forward(self.q, self.k, self.v, C=64, out=self.out, state_out=self.S,
                                   z_out=self.Z, workspace=self.ws)
        elif self.kind == "mg2":
            K.kata_mg_chunked_forward(self.q, self.k, self.v, g=2, C=64, out=self.out,
                                      state_out=self.S, z_out=self.Z, workspace=self.ws)
        else:
            K.kata_chunked_forward_from_state(self.q, self.k, self.v, self.S_in, self.Z_in, C=64,
                                              out=self.out, state_out=self.S, z_out=self.Z,
                                              workspace=self.ws)

    def results(self):
        return self.out.clone(), self.S.clone(), self.Z.clone()


# Rounding-order differences only.  An output entry whose final bf16
# rounding falls the other way moves by up to 2^-8 of itself, so 2^-7 of the
# row's largest entry allows that twice over; the fp32 state's sums, reordered,
# stay far inside 2^-16 of the tensor's largest entry.
OUT_REORDER = 2.0 ** -7
STATE_REORDER = 2.0 ** -16


def assert_same(got, want, what):
    out, ref = got[0].float(), want[0].float()
    row = ref.abs().amax(dim=-1, keepdim=True).clamp_min(1e-30)
    err = float(((out - ref).abs() / row).max())
    assert err <= OUT_REORDER, f"{what}: out differs from the call made on its own by {err:.2e}"
    for g, w, name in zip(got[1:], want[1:], ("S", "Z")):
        err = float((g - w).abs().max() / w.abs().max().clamp_min(1e-30))
        assert err <= STATE_REORDER, f"{what}: {name} differs from the call made on its own by {err:.2e}"


def inputs_for(B, H, T, d, seed):
    return inputs.make_qkv_device(B, H, T, d, d, seed=seed)


@pytest.mark.parametrize("kind,B,H,T,d", CASES)
def test_back_to_back_and_graph_replay(kind, B, H, T, d):
    c = Case(kind, B, H, T, d)
    xs = [inputs_for(B, H, T, d, seed=s) for s in (3, 4)]
    # each input on its own: the device idle before and after
    want = []
    for x in xs:
        c.load(x)
        c.out.fill_(float("nan"))
        c.S.fill_(float("nan"))
        c.Z.fill_(float("nan"))
        torch.cuda.synchronize()
        c.call()
        torch.cuda.synchronize()
        want.append(c.results())
    assert all(torch.isfinite(t).all() for t in want[0] + want[1])
    # the two inputs' results are far apart: a mix-up cannot pass
    with pytest.raises(AssertionError):
        assert_same(want[1], want[0], "the other input")

    # (a) alternating inputs, back to back on one stream, the same buffers;
    # each result copied out on the stream before the next call overwrites it
    got = []
    for i in range(6):
        c.load(xs[i % 2])
        c.call()
        got.append(c.results())
    torch.cuda.synchronize()
    for i, r in enumerate(got):
        assert_same(r, want[i % 2], f"back-to-back call {i}")

    # (b) the call captured once, replayed on each input
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        c.call()  # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        c.call()
    for i in range(4):
        c.load(xs[(i + 1) % 2])
        graph.replay()
        r = c.results()
        torch.cuda.synchronize()
        assert_same(r, want[(i + 1) % 2], f"graph replay {i}")
    del graph
