"""Write quintic_exact.json: exact rational values of the scalar quintic.

Newton-Schulz with odd polynomial f(s) = a s + b s^3 + c s^5 acts on each
singular value of the normalised matrix separately (DeMuon page, Method 1:
the iteration approximates msgn, which maps U S V^T to U V^T).  For inputs
whose singular values are known exactly (a row vector, a diagonal matrix)
the output is therefore f^k applied to those values.  This script evaluates
f^k exactly with Python fractions, independently of the matrix oracle and
of any floating-point library, and stores the results rounded to 17
significant digits.

Run: python tests/golden/make_quintic_exact.py
"""
import json
import os
from fractions import Fraction

COEFFS = (Fraction("3.4445"), Fraction("-4.7750"), Fraction("2.0315"))
CUBIC = (Fraction(3, 2), Fraction(-1, 2), Fraction(0))
POINTS = ["1", "3/5", "4/5", "1/3", "2/3", "1/10", "1/100", "1/2"]


def f(x, co):
    a, b, c = co
    return a * x + b * x ** 3 + c * x ** 5


def main():
    out = {
        "source": ("scalar Newton-Schulz polynomial f(s) = a s + b s^3 + c s^5 iterated 5 times, "
                   "exact in rationals; the iteration approximates msgn (DeMuon technical summary, "
                   "Methodology 1, matrix orthogonalisation) and acts on each singular value alone"),
        "generator": "tests/golden/make_quintic_exact.py",
        "coeffs": [str(c) for c in COEFFS],
        "quintic": {},
        "cubic": {},
    }
    for p in POINTS:
        x = Fraction(p)
        seq, y = [], x
        for _ in range(5):
            y = f(y, COEFFS)
            seq.append(format(float(y), ".17g"))
        out["quintic"][p] = seq
        seq, y = [], x
        for _ in range(5):
            y = f(y, CUBIC)
            seq.append(format(float(y), ".17g"))
        out["cubic"][p] = seq
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "quintic_exact.json")
    with open(path, "w") as fh:
        json.dump(out, fh, indent=1)
        fh.write("\n")


if __name__ == "__main__":
    main()
