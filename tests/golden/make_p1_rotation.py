"""Write ``p1_rotation_d2.txt``: the closed-form rotation of the d=2 worked example.

"Complex KDA ..." page, section "Complex KDA (CKDA) Mimarisi ve Parametre
Genislemesi" (and the "Kimi Delta Attention enhanced ..." page, first section):
one delta-rule step combined with the reflection supplied by the channel gate
gives a 2D rotation without raising the state rank.  Concretely, the gate
Diag(1, -1) followed by the beta = 2 Householder reflection about
k = (cos phi, sin phi) is the rotation R(2 phi + pi).

Values here come from the closed form only (cos and sin of 2 phi + pi); no
oracle or kernel code is called.
"""
import math
import os

PHIS = [0.0, math.pi / 6, math.pi / 4, math.pi / 3, math.pi / 2, 1.0, 2.5, -0.7, 3.0]


def main():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "p1_rotation_d2.txt")
    with open(path, "w") as f:
        f.write("# d=2 worked example: (I - 2 k k^T) Diag(1, -1) = R(2 phi + pi), k = (cos phi, sin phi)\n")
        f.write("# source: 'Complex KDA' page, section 'Complex KDA (CKDA) Mimarisi ve Parametre Genislemesi'\n")
        f.write("# columns: phi R00 R01 R10 R11   with R = [[cos t, -sin t], [sin t, cos t]], t = 2 phi + pi\n")
        for phi in PHIS:
            t = 2.0 * phi + math.pi
            c, s = math.cos(t), math.sin(t)
            f.write(f"{phi!r} {c!r} {-s!r} {s!r} {c!r}\n")


if __name__ == "__main__":
    main()
