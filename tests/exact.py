"""Exact-arithmetic witness for the GR-KAN activation, test-only.

Evaluates y = P(x) / (1 + |Q(x)|) in exact rational arithmetic with forward-
mode dual numbers, so every gradient (dx, dA, dB) comes from differentiating
the forward definition mechanically, not from a typed-in gradient formula.
The derivative of |q| at q = 0 is taken as 0 (the subgradient sign(0) = 0,
which is also what torch's abs backward uses).

Independent of ``oracle/``: it imports nothing from there.
"""
from fractions import Fraction


class Dual:
    __slots__ = ("v", "d")

    def __init__(self, v, d=0):
        self.v = Fraction(v)
        self.d = Fraction(d)

    @staticmethod
    def lift(o):
        return o if isinstance(o, Dual) else Dual(o)

    def __add__(self, o):
        o = Dual.lift(o)
        return Dual(self.v + o.v, self.d + o.d)

    __radd__ = __add__

    def __sub__(self, o):
        o = Dual.lift(o)
        return Dual(self.v - o.v, self.d - o.d)

    def __rsub__(self, o):
        return Dual.lift(o) - self

    def __mul__(self, o):
        o = Dual.lift(o)
        return Dual(self.v * o.v, self.v * o.d + self.d * o.v)

    __rmul__ = __mul__

    def __truediv__(self, o):
        o = Dual.lift(o)
        return Dual(self.v / o.v, (self.d * o.v - self.v * o.d) / (o.v * o.v))

    def __abs__(self):
        s = (self.v > 0) - (self.v < 0)
        return Dual(abs(self.v), s * self.d)


def activation(x, a, b):
    """y(x) for one element: a = [a_0..a_m], b = [b_1..b_n] (Duals or numbers)."""
    m = len(a) - 1
    P = Dual.lift(a[m])
    for i in range(m - 1, -1, -1):
        P = P * x + a[i]
    Q = Dual(0)
    xp = Dual.lift(x)
    for j in range(1, len(b) + 1):
        Q = Q + b[j - 1] * xp
        xp = xp * x
    return P / (1 + abs(Q))


def forward_backward(x, dy, a, b, n_g):
    """Exact y, dx (lists of rows) and dA, dB for a small (rows, d) case.

    x, dy: nested lists of numbers (rows x d); a: n_g lists of m+1; b: n_g lists of n.
    Returns Fractions."""
    rows, d = len(x), len(x[0])
    dg = d // n_g
    m1, n = len(a[0]), len(b[0])
    y = [[None] * d for _ in range(rows)]
    dx = [[None] * d for _ in range(rows)]
    dA = [[Fraction(0)] * m1 for _ in range(n_g)]
    dB = [[Fraction(0)] * n for _ in range(n_g)]
    for r in range(rows):
        for c in range(d):
            g = c // dg
            xv = Fraction(x[r][c])
            gv = Fraction(dy[r][c])
            ga = [Fraction(v) for v in a[g]]
            gb = [Fraction(v) for v in b[g]]
            # value and d/dx
            out = activation(Dual(xv, 1), ga, gb)
            y[r][c] = out.v
            dx[r][c] = gv * out.d
            # d/da_i, d/db_j, one seeded parameter at a time
            for i in range(m1):
                aa = [Dual(v, 1 if k == i else 0) for k, v in enumerate(ga)]
                dA[g][i] += gv * activation(Dual(xv), aa, gb).d
            for j in range(n):
                bb = [Dual(v, 1 if k == j else 0) for k, v in enumerate(gb)]
                dB[g][j] += gv * activation(Dual(xv), ga, bb).d
    return y, dx, dA, dB
