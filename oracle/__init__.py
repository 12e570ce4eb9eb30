"""CPU oracle of spatial sparse attention: test infrastructure only.

Imported by the tests, the package smoke check and the bench's CPU-baseline
leg; never by the library's product path.
"""
