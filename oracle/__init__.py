"""CPU oracle of the Token Radius Attention hot path (test infrastructure).

Only tests/, the smoke entry point and the bench's CPU-baseline leg use this
package.  It shares no code with the CUDA library and imports nothing from it.
"""
