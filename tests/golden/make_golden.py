"""Write the codebook fixtures in this folder from the CPU oracle (and nothing else).

Run from the repository root:  python tests/golden/make_golden.py
Each file holds one binary32 value per line as a hex float, preceded by '#' comment lines that
state the source the table is constructed from.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

SOURCES = {
    "code_dynamic_signed": (
        "source: dynamic (non-linear) quantization named in the abstract of Dettmers et al., "
        "'8-bit Optimizers via Block-wise Quantization' (arXiv 2110.02861), quoted on the page "
        "'Py之bitsandbytes：bitsandbytes的简介、安装、使用方法之详细攻略', section 2.\n"
        "reading: dynamic tree, sign + 7 magnitude bits, magnitude 10^-E * (0.1 + 0.9 (k+1)/2^(6-E)), "
        "E = 0..6, plus zero and +1e-7 in place of the negative zero.  256 values, ascending."),
    "code_dynamic_unsigned": (
        "source: as code_dynamic_signed (same abstract).\n"
        "reading: dynamic tree, 8 magnitude bits, 10^-E * (0.1 + 0.9 (k+1)/2^(7-E)), E = 0..7, plus zero. "
        "256 values, ascending."),
    "code_nf4": (
        "source: NF4 data type, page 'Bitsandbytes' (transformers docs), section 'Normal Float 4 (NF4)'; "
        "construction from Dettmers et al., 'QLoRA', section 3.\n"
        "reading: N(0,1) quantiles at probabilities delta + (1/2-delta) k/7 (k=0..6), zero, and "
        "1/2 + (1/2-delta) k/8 (k=1..8), divided by the largest; delta = (1/30 + 1/32)/2.  16 values."),
    "code_fp4": (
        "source: FP4 data type, page 'Quantize 🤗 Transformers models', section 'FP4 quantization'; "
        "format E2M1 of the OCP Microscaling Formats (MX) specification v1.0, section 5.3.3.\n"
        "reading: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 with both signs, divided by 6; the negative-zero "
        "pattern takes 0.25/6 so the table is strictly increasing.  16 values, ascending."),
    "code_linear": (
        "source: 'linear quantization' in the feature list of the page "
        "'Py之bitsandbytes：bitsandbytes的简介、安装、使用方法之详细攻略', section 1.\n"
        "reading: -1 + 2k/255, k = 0..255 (test table only)."),
}


def main():
    for name, src in SOURCES.items():
        vals = getattr(oracle, name)()
        with open(os.path.join(HERE, name + ".hex"), "w") as f:
            for line in src.splitlines():
                f.write("# " + line + "\n")
            f.write("# written by tests/golden/make_golden.py from the CPU oracle\n")
            for v in vals:
                f.write(float(v).hex() + "\n")
        print("wrote", name, len(vals))


if __name__ == "__main__":
    main()
