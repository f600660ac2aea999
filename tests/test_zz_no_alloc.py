"""q2_argmax_noalloc: the argmax entry point that allocates nothing.

Some callers cannot let a library allocate device memory while they call it
(a host that gives all device memory to its own pool, a loop that must not
wait on the allocator, code recording a CUDA graph under a capture mode that
refuses allocation).  This variant keeps its partials in a fixed array of the
library's device memory.  Checked here through the C ABI against the regular
q2_argmax and against the CPU oracle's argmax (first index of the maximum):
identical indices and values (bit-exact, the argmax tolerance of these
tests), on two calls in a row that share that array.  The file runs last so
that a stop-at-first-failure run has already run everything else.
"""

import pytest
import torch

import oracle
import qwen2_decode_step_b200 as q2
from synth import normal
from tol import bits_equal

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dt,rows,n", [("f32", 64, 151936), ("bf16", 3, 4097), ("f32", 1, 1)])
def test_noalloc_argmax_matches_argmax_and_the_oracle_on_two_calls_in_a_row(cuda_ok, dt, rows, n):
    tdt = torch.float32 if dt == "f32" else torch.bfloat16
    for call in range(2):
        x = normal((rows, n), 1.0, 500 + call, dt).cuda()
        if call == 1 and n > 10:
            x[0, 3] = x[0, n - 2] = x.max() + 1  # a tie: the lowest index must win
        ref_i = torch.empty(rows, dtype=torch.int64, device="cuda")
        ref_v = torch.empty(rows, dtype=tdt, device="cuda")
        q2.q2_argmax(ref_i, ref_v, x)
        got_i = torch.full((rows,), -1, dtype=torch.int64, device="cuda")
        got_v = torch.empty(rows, dtype=tdt, device="cuda")
        q2.q2_argmax_noalloc(got_i, got_v, x)
        torch.cuda.synchronize()
        assert torch.equal(got_i.cpu(), ref_i.cpu()), call
        assert bits_equal(got_v, ref_v), call
        o_i, o_v = oracle.argmax(x.cpu())
        assert torch.equal(got_i.cpu(), o_i), call
        assert bits_equal(got_v, o_v), call
        if call == 1 and n > 10:
            assert int(got_i[0]) == 3


def test_noalloc_argmax_rejects_too_many_rows(cuda_ok):
    x = torch.zeros((16385, 1), device="cuda")
    idx = torch.empty(16385, dtype=torch.int64, device="cuda")
    with pytest.raises(q2.Q2Error) as e:
        q2.q2_argmax_noalloc(idx, None, x)
    assert e.value.status == "Q2_ERR_CAPACITY"
