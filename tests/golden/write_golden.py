"""Write the derived expected values kept under tests/golden/.

Calls only the CPU oracle (``oracle.nf4_oracle``); nothing here touches the CUDA library.
Run from the repository root:  python tests/golden/write_golden.py

Outputs:
  nf4_codebook.txt   the 16 fp32 NF4 levels and 15 fp32 midpoints, as hex bit patterns
                     and decimal, derived from standard-normal quantiles ("QLoRA in LLMs"
                     section 5; "Idea one: NF4").
"""

from __future__ import annotations

import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import nf4_oracle as O  # noqa: E402


def main() -> None:
    q = O.nf4_codebook()
    m = O.nf4_midpoints(q)
    lines = ["# NF4 codebook derived by oracle/nf4_oracle.py (tests/golden/write_golden.py)",
             "# kind index hex_f32 decimal"]
    for i, v in enumerate(q):
        lines.append(f"level {i} 0x{int(np.float32(v).view(np.uint32)):08x} {float(v):.9g}")
    for i, v in enumerate(m):
        lines.append(f"mid {i} 0x{int(np.float32(v).view(np.uint32)):08x} {float(v):.9g}")
    with open(os.path.join(HERE, "nf4_codebook.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
