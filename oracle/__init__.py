"""CPU oracle for ADAMAS sparse decode attention -- test infrastructure only.

Only the tests, the package smoke check and the bench's CPU-baseline leg may
import anything here; the product path never does.
"""
