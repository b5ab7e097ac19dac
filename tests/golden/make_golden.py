"""Write the golden snapshot of the oracle on the tiny decode workload.

Calls only the oracle (and the seeded input generator). Run from the repository root:
    python tests/golden/make_golden.py
The workload: batch 2, pool of 4 slots, 4 heads, dim 16, dstate 16, one group, fp32
everything, softplus with dt_bias, no z, stateIndices [2, 0], seed 0 -- the single-token
decode of mamba_ssm::invokeSelectiveStateUpdate (Selective State Update page,
TensorRT-Edge-LLM C++ API).
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from linear_attention_recurrent_selective_b200.workloads import make_config  # noqa: E402
from oracle import oracle  # noqa: E402


def main():
    case = make_config("tiny_decode")
    out, pool, err = oracle.decode_case(case)
    assert err == 0
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_decode.txt")
    with open(path, "w") as f:
        f.write("# oracle snapshot: tiny decode workload (seed 0); see make_golden.py\n")
        f.write("# section out: [batch=2, H=4, Dm=16] float64, row-major\n")
        f.write("# section state: slots 2 and 0 after the step, [2, H=4, Dm=16, N=16] fp32\n")
        f.write("out\n")
        for v in out.reshape(-1).tolist():
            f.write(f"{v!r}\n")
        f.write("state\n")
        st = pool.view(4, -1)[[2, 0]].reshape(-1)
        for v in st.tolist():
            f.write(f"{v!r}\n")


if __name__ == "__main__":
    main()
